"""Shared set-up for the GPU parity tests: synthetic weights packed by the
library and, independently, quantized by the oracle from the same bf16
weights.  The oracle side never sees anything the CUDA path produced."""
from __future__ import annotations

import dataclasses

import numpy as np

from oracle import qmoe_oracle as Q
from skinny_gemm_top_b200 import synth

FMTS = {"int2": 2, "int4": 4, "ternary": 3}

# Tolerances: relative L2 error and max |err| / rms(ref) of the bf16 outputs.
REL_L2 = 5e-3
MAX_ERR_RMS = 3e-2


def block_scaled_weights(seed, rows, K, block, factors):
    """N(0, 0.02) bf16 weights whose 64/128-column blocks are multiplied by
    `factors` in turn: tiny blocks give tiny normal and subnormal bf16 scales."""
    w = synth.bf16_bits_to_f32(synth.normal_bf16(seed, 60, 99, (rows, K), 0.02))
    f = np.asarray(factors, dtype=np.float32)
    per_col = np.repeat(f[np.arange(K // block) % len(f)], block)
    return synth.f32_to_bf16_bits(w * per_col[None, :])


TINY_FACTORS = (1.0, 1e-30, 1e-36, 2e-37, 1e-38, 1e-39, 3e-40)


def to_dev(a: np.ndarray):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def bf16_dev_to_f64(t) -> np.ndarray:
    return Q.bf16_bits_to_f64(t.cpu().numpy().view(np.uint16))


def oracle_quant(fmt: str, w_bits: np.ndarray, block: int):
    w = Q.bf16_bits_to_f64(w_bits)
    if fmt == "ternary":
        return Q.quantize_ternary(w, block)
    return Q.quantize_sym(w, FMTS[fmt], block)


def oracle_quant_affine(fmt: str, w_bits: np.ndarray, block: int):
    return Q.quantize_affine(Q.bf16_bits_to_f64(w_bits), FMTS[fmt], block)


class MoECase:
    """A MoE layer: packed on the device for the library, quantized lazily by
    the oracle for reference values."""

    def __init__(self, cfg: synth.MoEConfig, seed: int = 1, affine: bool = False):
        from skinny_gemm_top_b200 import qmoe
        self.cfg, self.seed = cfg, seed
        n = cfg.E + cfg.n_shared
        f1, f2 = FMTS[cfg.fc1_fmt], FMTS[cfg.fc2_fmt]
        z1 = z2 = None
        if affine:  # scale and zero point per block (INT2 / INT4)
            c1, s1, z1 = qmoe.pack_stack_affine(f1, qmoe.ROWS_GATE_UP,
                                                (synth.expert_fc1(cfg, seed, e) for e in range(n)), cfg.block)
            c2, s2, z2 = qmoe.pack_stack_affine(f2, qmoe.ROWS_KSPLIT,
                                                (synth.expert_fc2(cfg, seed, e) for e in range(n)), cfg.block)
        else:
            c1, s1 = qmoe.pack_stack(f1, qmoe.ROWS_GATE_UP, (synth.expert_fc1(cfg, seed, e) for e in range(n)),
                                     cfg.block)
            c2, s2 = qmoe.pack_stack(f2, qmoe.ROWS_KSPLIT, (synth.expert_fc2(cfg, seed, e) for e in range(n)),
                                     cfg.block)
        self.dev = {"c1": to_dev(c1), "s1": to_dev(s1), "c2": to_dev(c2), "s2": to_dev(s2)}
        if affine:
            self.dev["z1"], self.dev["z2"] = to_dev(z1), to_dev(z2)
        self.b1 = self.b2 = None
        if cfg.bias:
            self.dev["b1"] = to_dev(np.stack([synth.expert_b1(cfg, seed, e) for e in range(n)]))
            self.dev["b2"] = to_dev(np.stack([synth.expert_b2(cfg, seed, e) for e in range(n)]))
        self.w1 = qmoe.make_weights(f1, cfg.block, self.dev["c1"], self.dev["s1"], self.dev.get("b1"), qmoe.ROWS_GATE_UP,
                                    self.dev.get("z1"))
        self.w2 = qmoe.make_weights(f2, cfg.block, self.dev["c2"], self.dev["s2"], self.dev.get("b2"), qmoe.ROWS_KSPLIT,
                                    self.dev.get("z2"))
        quant = oracle_quant_affine if affine else oracle_quant
        self.bank = Q.QuantExpertBank(
            cfg.H, cfg.I, cfg.E, cfg.n_shared, cfg.block,
            lambda e: quant(cfg.fc1_fmt, synth.expert_fc1(cfg, seed, e), cfg.block),
            lambda e: quant(cfg.fc2_fmt, synth.expert_fc2(cfg, seed, e), cfg.block),
            (lambda e: Q.bf16_bits_to_f64(synth.expert_b1(cfg, seed, e))) if cfg.bias else None,
            (lambda e: Q.bf16_bits_to_f64(synth.expert_b2(cfg, seed, e))) if cfg.bias else None,
            cache=16)

    def layer(self, path=0, max_row_tile=0):
        from skinny_gemm_top_b200 import qmoe
        c = self.cfg
        return qmoe.make_layer(c.H, c.I, c.E, c.k, c.n_shared, self.w1, self.w2, path, max_row_tile)

    def run(self, x_bits: np.ndarray, logits: np.ndarray, ws_bytes: int | None = None, max_row_tile: int = 0,
            path: int = 0):
        import torch
        from skinny_gemm_top_b200 import qmoe
        T = x_bits.shape[0]
        layer = self.layer(path=path, max_row_tile=max_row_tile)
        need = qmoe.workspace_size(layer, T)
        ws = torch.empty(need if ws_bytes is None else ws_bytes, dtype=torch.uint8, device="cuda")
        x = to_dev(x_bits)
        lg = torch.from_numpy(np.ascontiguousarray(logits, dtype=np.float32)).cuda()
        y = torch.empty((T, self.cfg.H), dtype=torch.int16, device="cuda")
        qmoe.forward(layer, x, lg, y, ws)
        torch.cuda.synchronize()
        return bf16_dev_to_f64(y)


def small_cfg(base: synth.MoEConfig, **kw) -> synth.MoEConfig:
    return dataclasses.replace(base, **kw)


class ChanCase:
    """A channel layer (top-k channel-selective read): channel records and
    sketches packed by the library on the host, and, independently, the
    oracle's bank built from the same bf16 weights and signs."""

    def __init__(self, cfg: synth.MoEConfig, seed: int = 1):
        import torch
        from oracle import channel_select as CS
        from skinny_gemm_top_b200 import qmoe
        self.cfg, self.seed = cfg, seed
        f1, f2 = FMTS[cfg.fc1_fmt], FMTS[cfg.fc2_fmt]
        self.signs = synth.rht_signs(seed, cfg.H)
        recs, sks, dns = [], [], []
        for e in range(cfg.E + cfg.n_shared):
            routed = e < cfg.E
            r, s, d = qmoe.chan_pack(f1, f2, synth.expert_fc1(cfg, seed, e), synth.expert_fc2(cfg, seed, e),
                                     cfg.block, self.signs if routed else None, sketch=routed)
            recs.append(r)
            if routed:
                sks.append(s)
                dns.append(d)
        self.dev = {"rec": to_dev(np.concatenate(recs)), "sk": to_dev(np.concatenate(sks)),
                    "dn": torch.from_numpy(np.concatenate(dns)).cuda(), "signs": torch.from_numpy(self.signs).cuda()}
        self.layer = qmoe.make_chan_layer(cfg.H, cfg.I, cfg.E, cfg.k, cfg.n_shared, f1, f2, cfg.block,
                                          self.dev["rec"], self.dev["sk"], self.dev["dn"], self.dev["signs"])
        self.bank = CS.ChannelExpertBank(
            cfg.H, cfg.I, cfg.E, cfg.n_shared, cfg.block, f1, f2,
            lambda e: Q.bf16_bits_to_f64(synth.expert_fc1(cfg, seed, e)),
            lambda e: Q.bf16_bits_to_f64(synth.expert_fc2(cfg, seed, e)), self.signs)

    def run(self, x_bits: np.ndarray, logits: np.ndarray, n_keep: int, ws_bytes: int | None = None):
        """(y float64 [T, H], sel [T, n_keep], scores float32 [T, k * I]) from the device."""
        import torch
        from skinny_gemm_top_b200 import qmoe
        T, c = x_bits.shape[0], self.cfg
        need = qmoe.chan_workspace_size(self.layer, T, n_keep)
        ws = torch.empty(need if ws_bytes is None else ws_bytes, dtype=torch.uint8, device="cuda")
        x = to_dev(x_bits)
        lg = torch.from_numpy(np.ascontiguousarray(logits, dtype=np.float32)).cuda()
        y = torch.empty((T, c.H), dtype=torch.int16, device="cuda")
        sel = torch.full((T, max(n_keep, 1)), -1, dtype=torch.int32, device="cuda")
        sc = torch.empty((T, c.k * c.I), dtype=torch.float32, device="cuda")
        qmoe.chan_forward(self.layer, x, lg, n_keep, y, ws, sel=sel, scores=sc)
        torch.cuda.synchronize()
        return bf16_dev_to_f64(y), sel.cpu().numpy()[:, :n_keep], sc.cpu().numpy()
