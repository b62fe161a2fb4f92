// Top-k channel-selective MoE layer: kernels.
//
// "Skip MoE channels for up to 2.69x faster MoE blocks - top-k channel
// selection" explainer: a ternary sketch of the randomized-Hadamard-rotated
// gate and up rows estimates every channel's activation (sketch paragraph); a
// channel's score is router weight x down-column norm x |estimate|, channels
// of all routed experts compete in one top-k, and the winners are read in
// full and computed exactly (scoring paragraph); the number of channels read
// per token is fixed (choosing-k paragraph).  Shared experts are read in full.
//
// Three launches, chained by programmatic dependent launch:
//   chan_score_kernel   routing, rotation of x, sketch products, scores
//   chan_select_kernel  one block per token: radix select of the n_keep best
//   chan_exact_kernel   the selected and shared channel records: gate/up dot
//                       products, SwiGLU, down-column accumulation, combine
//
// A channel (and its sketch) is one contiguous record, so a block's work is a
// list of records streamed into shared memory with 16-byte cp.async by every
// thread, completing on one mbarrier per wave.  The dot products run on the
// CUDA cores: a code u is turned into the float 1 + u / 2^bits' (one shift and
// one LOP3 into the mantissa), multiplied with x, and the constant part is
// removed with the per-chunk sum of x.
#pragma once
#include <climits>
#include <cmath>
#include <type_traits>

#include "device_common.cuh"
#include "qmm_small.cuh"  // silu_f

namespace qmoe {

constexpr int kChanThreads = 512;
constexpr int kChanWarps = kChanThreads / 32;
constexpr int kChanMaxT = 8;
constexpr int kChanMaxK = 8;
constexpr int kChanMaxAct = kChanMaxT * kChanMaxK;
constexpr int kSelThreads = 1024;
constexpr int kChanMaxCand = 32768;  // k * I of one token (selection block's shared memory)
constexpr int kSketchBlock = 128;

struct ChanParams {
  int H, I, E, k, S, T;  // S shared experts (stored after the E routed ones)
  int fmt1, fmt2, block;
  int rec_bytes, sk_bytes;
  const uint8_t* rec;     // [E + S][I] channel records
  const uint8_t* sketch;  // [E][I] sketch records
  const float* dn;        // [E][I] down-column norms
  const float* signs;     // [H] rotation signs
  const uint16_t* x;      // [T][H] bf16
  const float* logits;    // [T][E]
  int n_keep;
  int* ids;               // [T][k] routed experts
  float* wts;             // [T][k] router weights
  float* scores;          // [T][k * I]
  int* sel;               // [T][n_keep] selected flat indices s * I + j, ascending
  float* yacc;            // [T][H] fp32 accumulator, zeroed by the score kernel
  int* ticket;            // [0] exact-kernel blocks done, [1] blocks that gave up
  uint16_t* y;            // [T][H] bf16
  float inv_sqrt_h;       // 1 / sqrt(H)
  int wave_sk;            // sketch records per wave of the score kernel
  int wave_rec;           // channel records per wave of the exact kernel
  unsigned long long wait_ns;
  unsigned* status;
};

// ---------------------------------------------------------------------------
// Routing of one token by one warp: top-k of the fp32 logits by repeated warp
// argmax (ties to the lower expert), then a softmax over the k selected, in
// slot order.  E <= 256.
__device__ __forceinline__ void chan_route_token(const float* lg, int E, int k, int lane, int* ids, float* w) {
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? lg[e] : -INFINITY;
  }
  unsigned taken = 0;
  float lsel[kChanMaxK];
  int esel[kChanMaxK];
#pragma unroll
  for (int s = 0; s < kChanMaxK; ++s) {
    lsel[s] = -INFINITY;
    esel[s] = 0;
    if (s < k) {
      float bv = -INFINITY;
      int be = INT_MAX;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !((taken >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < be))) {
          bv = v[i];
          be = e;
        }
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oe = __shfl_xor_sync(0xffffffffu, be, off);
        if (ov > bv || (ov == bv && oe < be)) {
          bv = ov;
          be = oe;
        }
      }
      if (be == INT_MAX) be = 0;  // fewer than k finite candidates: not reached for E >= k
      if ((be & 31) == lane) taken |= 1u << (be >> 5);
      lsel[s] = bv;
      esel[s] = be;
    }
  }
  if (lane == 0) {
    float z[kChanMaxK], sum = 0.f;
#pragma unroll
    for (int s = 0; s < kChanMaxK; ++s)
      if (s < k) {
        z[s] = expf(lsel[s] - lsel[0]);
        sum += z[s];
      }
#pragma unroll
    for (int s = 0; s < kChanMaxK; ++s)
      if (s < k) {
        ids[s] = esel[s];
        w[s] = z[s] / sum;
      }
  }
}

// Float 1 + u / 4 of the 2-bit field k of w (a trit t = u - 2 of the sketch).
template <int K>
__device__ __forceinline__ float code2_f(uint32_t w) {
  const uint32_t s = 2 * K <= 21 ? (w << (21 - 2 * K)) : (w >> (2 * K - 21));
  return __uint_as_float(lop3_and_or(s, 0x00600000u, 0x3F800000u));
}
// Float 1 + u / 16 of the 4-bit field k of w.
template <int K>
__device__ __forceinline__ float code4_f(uint32_t w) {
  const uint32_t s = 4 * K <= 19 ? (w << (19 - 4 * K)) : (w >> (4 * K - 19));
  return __uint_as_float(lop3_and_or(s, 0x00780000u, 0x3F800000u));
}

template <int N>
struct Unroll {
  template <typename F>
  __device__ __forceinline__ static void run(F&& f) {
    Unroll<N - 1>::run(f);
    f(std::integral_constant<int, N - 1>());
  }
};
template <>
struct Unroll<0> {
  template <typename F>
  __device__ __forceinline__ static void run(F&&) {}
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Balanced split of n units over the grid.
__device__ __forceinline__ void chan_range(int n, int* lo, int* hi) {
  *lo = (int)((long long)n * blockIdx.x / gridDim.x);
  *hi = (int)((long long)n * (blockIdx.x + 1) / gridDim.x);
}

// All threads: copy `n` records of `bytes` bytes (sources in src[]) into buf
// with 16-byte cp.async, then arrive on bar (count kChanThreads) when this
// thread's copies have landed.
__device__ __forceinline__ void chan_copy_wave(uint8_t* buf, const uint8_t* const* src, int n, int bytes,
                                               uint64_t* bar) {
  const int per = bytes / 16;
  const int total = n * per;
  for (int c = threadIdx.x; c < total; c += kChanThreads) {
    const int i = c / per, o = c - i * per;
    cp_async16(buf + (size_t)i * bytes + 16 * o, src[i] + 16 * o);
  }
  cp_async_arrive(bar);
}

// ---------------------------------------------------------------------------
// Scores.  Units: (active expert a, channel j), a over the distinct routed
// experts of the batch in ascending id; every token routed to a gets the
// score of channel j from one read of its sketch record.
//
// Shared memory: x' [T][4][H/16] float4 (word-interleaved: element c at word
// c / 16, quarter (c / 4) % 4, component c % 4), per-word sums of x' [T][H/16],
// record sources, then the wave of sketch records.
__global__ void __launch_bounds__(kChanThreads, 1) chan_score_kernel(ChanParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t bar;
  __shared__ int s_ids[kChanMaxAct];
  __shared__ float s_w[kChanMaxAct];
  __shared__ int s_act_e[kChanMaxAct], s_act_n[kChanMaxAct], s_act_m[kChanMaxAct][kChanMaxT];
  __shared__ int s_nact, s_abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H, W16 = H / 16, T = p.T, I = p.I, k = p.k;
  float* xs = reinterpret_cast<float*>(smem);
  float* sxw = xs + (size_t)T * H;
  const uint8_t** src =
      reinterpret_cast<const uint8_t**>((reinterpret_cast<uintptr_t>(sxw + (size_t)T * W16) + 15) & ~uintptr_t(15));
  uint8_t* buf = reinterpret_cast<uint8_t*>(src + p.wave_sk);
  buf = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(buf) + 127) & ~uintptr_t(127));

  if (tid == 0) {
    mbar_init(&bar, kChanThreads);
    fence_mbar_init();
    s_abort = 0;
  }
  pdl_wait();
  pdl_trigger();
  // the exact kernel's accumulator and tickets: its previous use has ended
  for (int i = blockIdx.x * kChanThreads + tid; i < T * H; i += gridDim.x * kChanThreads) p.yacc[i] = 0.f;
  if (blockIdx.x == 0 && tid < 2) p.ticket[tid] = 0;

  if (warp < T) chan_route_token(p.logits + (size_t)warp * p.E, p.E, k, lane, s_ids + warp * k, s_w + warp * k);
  __syncthreads();
  if (blockIdx.x == 0 && tid < T * k) {
    p.ids[tid] = s_ids[tid];
    p.wts[tid] = s_w[tid];
  }
  if (tid == 0) {  // distinct experts, ascending, each with its (token, slot) members in token order
    int n = 0;
    for (int m = 0; m < T * k; ++m) {
      const int e = s_ids[m];
      int a = 0;
      while (a < n && s_act_e[a] != e) ++a;
      if (a == n) {
        s_act_e[n] = e;
        s_act_n[n] = 0;
        ++n;
      }
      s_act_m[a][s_act_n[a]++] = m;
    }
    for (int a = 1; a < n; ++a)
      for (int b = a; b > 0 && s_act_e[b - 1] > s_act_e[b]; --b) {
        int te = s_act_e[b];
        s_act_e[b] = s_act_e[b - 1];
        s_act_e[b - 1] = te;
        int tn = s_act_n[b];
        s_act_n[b] = s_act_n[b - 1];
        s_act_n[b - 1] = tn;
        for (int q = 0; q < kChanMaxT; ++q) {
          int tm = s_act_m[b][q];
          s_act_m[b][q] = s_act_m[b - 1][q];
          s_act_m[b - 1][q] = tm;
        }
      }
    s_nact = n;
  }
  __syncthreads();
  int u0, u1;
  chan_range(s_nact * I, &u0, &u1);
  const int skb = p.sk_bytes;

  auto issue = [&](int w0, int nw) {
    for (int i = tid; i < nw; i += kChanThreads) {
      const int u = w0 + i, a = u / I, j = u - a * I;
      src[i] = p.sketch + ((size_t)s_act_e[a] * I + j) * skb;
    }
    __syncthreads();
    chan_copy_wave(buf, src, nw, skb, &bar);
  };
  if (u0 < u1) issue(u0, min(p.wave_sk, u1 - u0));

  // x' = Had (d * x) in place, unscaled (1/sqrt(H) is applied to the products)
  auto xi = [&](int t, int c) { return (((size_t)t * 4 + ((c >> 2) & 3)) * W16 + (c >> 4)) * 4 + (c & 3); };
  for (int i = tid; i < T * H; i += kChanThreads) {
    const int t = i / H, c = i - t * H;
    xs[xi(t, c)] = bf16_to_f(p.x[(size_t)t * H + c]) * p.signs[c];
  }
  for (int len = 1; len < H; len <<= 1) {
    __syncthreads();
    for (int b = tid; b < T * (H / 2); b += kChanThreads) {
      const int t = b / (H / 2), bb = b - t * (H / 2);
      const int i = (bb / len) * 2 * len + (bb % len);
      const size_t ia = xi(t, i), ib = xi(t, i + len);
      const float a = xs[ia], c = xs[ib];
      xs[ia] = a + c;
      xs[ib] = a - c;
    }
  }
  __syncthreads();
  for (int i = tid; i < T * W16; i += kChanThreads) {
    const int t = i / W16, w = i - t * W16;
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = reinterpret_cast<const float4*>(xs)[((size_t)t * 4 + q) * W16 + w];
      s += (v.x + v.y) + (v.z + v.w);
    }
    sxw[i] = s;
  }
  __syncthreads();

  const float4* x4 = reinterpret_cast<const float4*>(xs);
  const int SKB = H / kSketchBlock;
  int wave = 0;
  for (int w0 = u0; w0 < u1; w0 += p.wave_sk, ++wave) {
    const int nw = min(p.wave_sk, u1 - w0);
    if (w0 != u0) issue(w0, nw);
    if (!mbar_wait_sleep_bounded(&bar, wave & 1, p.status, p.wait_ns)) s_abort = 1;
    __syncthreads();
    if (s_abort) break;
    for (int i = warp; i < nw; i += kChanWarps) {
      const int u = w0 + i, a = u / I, j = u - a * I;
      const int nm = s_act_n[a];
      const uint8_t* r = buf + (size_t)i * skb;
      const uint32_t* gw = reinterpret_cast<const uint32_t*>(r);
      const uint32_t* uw = gw + W16;
      const uint16_t* sc = reinterpret_cast<const uint16_t*>(r + H / 2);
      int tok[kChanMaxT];
#pragma unroll
      for (int m = 0; m < kChanMaxT; ++m) tok[m] = m < nm ? s_act_m[a][m] / k : 0;
      float ag[kChanMaxT], au[kChanMaxT];
#pragma unroll
      for (int m = 0; m < kChanMaxT; ++m) ag[m] = au[m] = 0.f;
      for (int w = lane; w < W16; w += 32) {
        const uint32_t g = gw[w], uu = uw[w];
        const float sg = bf16_to_f(sc[w >> 3]), su = bf16_to_f(sc[SKB + (w >> 3)]);
        float vg[16], vu[16];
        Unroll<16>::run([&](auto kk) {
          constexpr int K = decltype(kk)::value;
          vg[K] = code2_f<K>(g);
          vu[K] = code2_f<K>(uu);
        });
#pragma unroll
        for (int m = 0; m < kChanMaxT; ++m) {
          if (m < nm) {
            const int t = tok[m];
            float dg = 0.f, du = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4 xv = x4[((size_t)t * 4 + q) * W16 + w];
              dg = fmaf(vg[4 * q], xv.x, dg);
              dg = fmaf(vg[4 * q + 1], xv.y, dg);
              dg = fmaf(vg[4 * q + 2], xv.z, dg);
              dg = fmaf(vg[4 * q + 3], xv.w, dg);
              du = fmaf(vu[4 * q], xv.x, du);
              du = fmaf(vu[4 * q + 1], xv.y, du);
              du = fmaf(vu[4 * q + 2], xv.z, du);
              du = fmaf(vu[4 * q + 3], xv.w, du);
            }
            const float sx = 6.f * sxw[t * W16 + w];
            ag[m] = fmaf(sg, fmaf(4.f, dg, -sx), ag[m]);
            au[m] = fmaf(su, fmaf(4.f, du, -sx), au[m]);
          }
        }
      }
      const int e = s_act_e[a];
      const float dnj = p.dn[(size_t)e * I + j];
#pragma unroll
      for (int m = 0; m < kChanMaxT; ++m) {
        if (m < nm) {
          const float gs = warp_sum(ag[m]) * p.inv_sqrt_h, us = warp_sum(au[m]) * p.inv_sqrt_h;
          if (lane == m) {
            const int mm = s_act_m[a][m], t = mm / k, s = mm - t * k;
            p.scores[((size_t)t * k + s) * I + j] = s_w[mm] * dnj * fabsf(silu_f(gs) * us);
          }
        }
      }
    }
    __syncthreads();  // the wave buffer is reused
  }
  if (s_abort) cp_async_wait_all();
}

// ---------------------------------------------------------------------------
// Selection: block t finds the n_keep best scores of token t (score
// descending, ties to the lower flat index) by a 4-pass 8-bit radix select on
// the score bits (scores are >= 0, so their bit patterns order like the
// values), then writes the selected indices in ascending order.
__device__ __forceinline__ void block_scan2(int a, int b, int* ea, int* eb, int* sh) {
  // exclusive prefix sums over the block of (a, b); sh: 2 * 32 ints
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int ia = a, ib = b;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int ta = __shfl_up_sync(0xffffffffu, ia, off), tb = __shfl_up_sync(0xffffffffu, ib, off);
    if (lane >= off) {
      ia += ta;
      ib += tb;
    }
  }
  if (lane == 31) {
    sh[warp] = ia;
    sh[32 + warp] = ib;
  }
  __syncthreads();
  if (warp == 0) {
    int va = lane < nw ? sh[lane] : 0, vb = lane < nw ? sh[32 + lane] : 0;
    const int oa = va, ob = vb;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int ta = __shfl_up_sync(0xffffffffu, va, off), tb = __shfl_up_sync(0xffffffffu, vb, off);
      if (lane >= off) {
        va += ta;
        vb += tb;
      }
    }
    sh[lane] = va - oa;
    sh[32 + lane] = vb - ob;
  }
  __syncthreads();
  *ea = sh[warp] + ia - a;
  *eb = sh[32 + warp] + ib - b;
  __syncthreads();
}

__global__ void __launch_bounds__(kSelThreads, 1) chan_select_kernel(ChanParams p) {
  extern __shared__ __align__(16) uint32_t keys[];
  __shared__ int hist[256];
  __shared__ int sh[64];
  __shared__ int s_b, s_above;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t = blockIdx.x, n = p.k * p.I;
  if (tid == 0) s_b = s_above = 0;
  pdl_wait();
  pdl_trigger();
  const float* sc = p.scores + (size_t)t * n;
  for (int i = tid; i < n; i += kSelThreads) keys[i] = __float_as_uint(sc[i]) & 0x7FFFFFFFu;
  uint32_t prefix = 0, pmask = 0;
  int need = p.n_keep;  // rank of the threshold among the keys that match the prefix
  for (int d = 3; d >= 0; --d) {
    for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kSelThreads) {
      const uint32_t key = keys[i];
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> (8 * d)) & 255u], 1);
    }
    __syncthreads();
    if (warp == 0) {  // lane l holds buckets 255 - 8l down to 248 - 8l
      int c[8], tot = 0;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        c[m] = hist[255 - 8 * lane - m];
        tot += c[m];
      }
      int incl = tot;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      const int excl = incl - tot;
      if (excl < need && need <= incl) {
        int run = excl;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          if (run + c[m] >= need) {
            s_b = 255 - 8 * lane - m;
            s_above = run;
            break;
          }
          run += c[m];
        }
      }
    }
    __syncthreads();
    need -= s_above;
    prefix |= (uint32_t)s_b << (8 * d);
    pmask |= 255u << (8 * d);
    __syncthreads();
  }
  const uint32_t theta = prefix;  // key of the n_keep-th best; `need` keys equal to it are taken
  const int per = (n + kSelThreads - 1) / kSelThreads;
  const int lo = min(n, tid * per), hi = min(n, lo + per);
  int gt = 0, eq = 0;
  for (int i = lo; i < hi; ++i) {
    gt += keys[i] > theta;
    eq += keys[i] == theta;
  }
  int gt0, eq0;
  block_scan2(gt, eq, &gt0, &eq0, sh);
  need = max(need, 0);
  int pos = gt0 + min(eq0, need), eqs = eq0;
  int* out = p.sel + (size_t)t * p.n_keep;
  for (int i = lo; i < hi; ++i) {
    const uint32_t key = keys[i];
    if ((key > theta || (key == theta && eqs++ < need)) && pos < p.n_keep) out[pos++] = i;
  }
}

// ---------------------------------------------------------------------------
// Exact read.  Units: the shared experts' channels (every token, weight 1),
// then the selected channels of each token (that token, its router weight).
// Per wave: FC1 with one warp per record (gate and up dot products over the
// record's 16-byte chunks, lane-strided), h = w * silu(g) * u into shared
// memory; then FC2 with each warp owning H / 16 output rows for every record
// of the wave, accumulated in registers; at the end the block's rows are added
// into yacc and the last block rounds y to bf16.
template <int F1, int F2, int TM>
__global__ void __launch_bounds__(kChanThreads, 1) chan_exact_kernel(ChanParams p) {
  constexpr int CPC = 128 / F1;          // columns per 16-byte chunk of a gate/up row
  constexpr int CPW = 32 / F1;           // columns per 32-bit word
  constexpr float kA = F1 == 4 ? 16.f : 4.f;               // sum c x = kA * sum v x - kB * sum x
  constexpr float kB = F1 == 4 ? 24.f : 6.f;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t bar;
  __shared__ int s_last, s_abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H, T = p.T, I = p.I, NC = H / CPC, R = p.rec_bytes, WR = p.wave_rec;
  const int SB = H / p.block;
  const int off_u = H * F1 / 8, off_d = 2 * off_u, off_s = off_d + H * F2 / 8;
  float* xs = reinterpret_cast<float*>(smem);                       // [T][CPC/4][NC] float4
  float* sxc = xs + (size_t)T * H;                                  // [T][NC]
  float* hc = sxc + (size_t)T * NC;                                 // [WR][TM]
  int* utok = reinterpret_cast<int*>(hc + (size_t)WR * TM);  // [WR]: token, or -1 for all
  float* uw = reinterpret_cast<float*>(utok + WR);                  // [WR]: weight
  uintptr_t sp = reinterpret_cast<uintptr_t>(uw + WR);
  const uint8_t** src = reinterpret_cast<const uint8_t**>((sp + 15) & ~uintptr_t(15));
  uint8_t* buf = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(src + WR) + 127) & ~uintptr_t(127));

  if (tid == 0) {
    mbar_init(&bar, kChanThreads);
    fence_mbar_init();
    s_abort = 0;
  }
  pdl_wait();
  pdl_trigger();
  for (int i = tid; i < T * H; i += kChanThreads) {
    const int t = i / H, c = i - t * H;
    const int ch = c / CPC, q = (c % CPC) >> 2;
    xs[(((size_t)t * (CPC / 4) + q) * NC + ch) * 4 + (c & 3)] = bf16_to_f(p.x[(size_t)t * H + c]);
  }
  __syncthreads();
  const float4* x4 = reinterpret_cast<const float4*>(xs);
  for (int i = tid; i < T * NC; i += kChanThreads) {
    const int t = i / NC, ch = i - t * NC;
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < CPC / 4; ++q) {
      const float4 v = x4[((size_t)t * (CPC / 4) + q) * NC + ch];
      s += (v.x + v.y) + (v.z + v.w);
    }
    sxc[i] = s;
  }

  const int n_sh = p.S * I;
  int u0, u1;
  chan_range(n_sh + T * p.n_keep, &u0, &u1);
  const int RPL = H / 512;  // output rows per lane in FC2 (1..8)
  const int r0 = warp * (H / 16) + lane * RPL;
  float acc[8][TM];
#pragma unroll
  for (int q = 0; q < 8; ++q)
#pragma unroll
    for (int t = 0; t < TM; ++t) acc[q][t] = 0.f;

  int wave = 0;
  for (int w0 = u0; w0 < u1; w0 += WR, ++wave) {
    const int nw = min(WR, u1 - w0);
    for (int i = tid; i < nw; i += kChanThreads) {
      const int u = w0 + i;
      int e, j, tok;
      float wt;
      if (u < n_sh) {
        e = p.E + u / I;
        j = u % I;
        tok = -1;
        wt = 1.f;
      } else {
        const int v = u - n_sh, t = v / p.n_keep;
        const int f = p.sel[v];
        const int s = f / I;
        e = (f >= 0 && s < p.k) ? p.ids[t * p.k + s] : -1;
        j = f - s * I;
        tok = t;
        wt = e >= 0 ? p.wts[t * p.k + s] : 0.f;
        if (e < 0 || e >= p.E) {  // a corrupt selection: read record 0, add nothing
          atomicOr(p.status, kStatusBadSegment);
          e = 0;
          j = 0;
          wt = 0.f;
        }
      }
      src[i] = p.rec + ((size_t)e * I + j) * R;
      utok[i] = tok;
      uw[i] = wt;
    }
    __syncthreads();
    chan_copy_wave(buf, src, nw, R, &bar);
    if (!mbar_wait_sleep_bounded(&bar, wave & 1, p.status, p.wait_ns)) s_abort = 1;
    __syncthreads();
    if (s_abort) break;

    // FC1: one warp per record
    for (int i = warp; i < nw; i += kChanWarps) {
      const uint8_t* r = buf + (size_t)i * R;
      const uint16_t* sc = reinterpret_cast<const uint16_t*>(r + off_s);
      const int tok = utok[i];
      const int nt = tok < 0 ? T : 1;
      float ag[TM], au[TM];
#pragma unroll
      for (int m = 0; m < TM; ++m) ag[m] = au[m] = 0.f;
      for (int ch = lane; ch < NC; ch += 32) {
        const uint4 G = *reinterpret_cast<const uint4*>(r + 16 * ch);
        const uint4 U = *reinterpret_cast<const uint4*>(r + off_u + 16 * ch);
        const int blk = ch * CPC / p.block;
        const float sg = bf16_to_f(sc[blk]), su = bf16_to_f(sc[SB + blk]);
        const uint32_t gw[4] = {G.x, G.y, G.z, G.w}, uwd[4] = {U.x, U.y, U.z, U.w};
        float dg[TM], du[TM];
#pragma unroll
        for (int m = 0; m < TM; ++m) dg[m] = du[m] = 0.f;
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
          float vg[CPW], vu[CPW];
          Unroll<CPW>::run([&](auto kk) {
            constexpr int K = decltype(kk)::value;
            if constexpr (F1 == 4) {
              vg[K] = code4_f<K>(gw[wd]);
              vu[K] = code4_f<K>(uwd[wd]);
            } else {
              vg[K] = code2_f<K>(gw[wd]);
              vu[K] = code2_f<K>(uwd[wd]);
            }
          });
#pragma unroll
          for (int m = 0; m < TM; ++m) {
            if (m < nt) {
              const int t = tok < 0 ? m : tok;
#pragma unroll
              for (int qq = 0; qq < CPW / 4; ++qq) {
                const float4 xv = x4[((size_t)t * (CPC / 4) + wd * (CPW / 4) + qq) * NC + ch];
                dg[m] = fmaf(vg[4 * qq], xv.x, dg[m]);
                dg[m] = fmaf(vg[4 * qq + 1], xv.y, dg[m]);
                dg[m] = fmaf(vg[4 * qq + 2], xv.z, dg[m]);
                dg[m] = fmaf(vg[4 * qq + 3], xv.w, dg[m]);
                du[m] = fmaf(vu[4 * qq], xv.x, du[m]);
                du[m] = fmaf(vu[4 * qq + 1], xv.y, du[m]);
                du[m] = fmaf(vu[4 * qq + 2], xv.z, du[m]);
                du[m] = fmaf(vu[4 * qq + 3], xv.w, du[m]);
              }
            }
          }
        }
#pragma unroll
        for (int m = 0; m < TM; ++m) {
          if (m < nt) {
            const float sx = kB * sxc[(tok < 0 ? m : tok) * NC + ch];
            ag[m] = fmaf(sg, fmaf(kA, dg[m], -sx), ag[m]);
            au[m] = fmaf(su, fmaf(kA, du[m], -sx), au[m]);
          }
        }
      }
      const float wt = uw[i];
      if (tok < 0) {  // a shared expert: every token
#pragma unroll
        for (int m = 0; m < TM; ++m) {
          float h = 0.f;
          if (m < T) h = wt * silu_f(warp_sum(ag[m])) * warp_sum(au[m]);
          if (lane == 0) hc[i * TM + m] = h;
        }
      } else {
        const float h = wt * silu_f(warp_sum(ag[0])) * warp_sum(au[0]);
        if (lane == 0)
#pragma unroll
          for (int m = 0; m < TM; ++m) hc[i * TM + m] = m == tok ? h : 0.f;
      }
    }
    __syncthreads();

    // FC2: warp rows [warp * H / 16, (warp + 1) * H / 16), RPL consecutive rows per lane
    {
      const uint16_t* sdn = nullptr;
      for (int i = 0; i < nw; ++i) {
        const uint8_t* r = buf + (size_t)i * R;
        sdn = reinterpret_cast<const uint16_t*>(r + off_s) + 2 * SB;
        const uint32_t wd = reinterpret_cast<const uint32_t*>(r + off_d)[(r0 * F2) >> 5] >> ((r0 * F2) & 31);
        const float sd = bf16_to_f(sdn[r0 / p.block]);
        float hv[TM];
#pragma unroll
        for (int t = 0; t < TM; ++t) hv[t] = t < T ? hc[i * TM + t] : 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (q < RPL) {
            const float d = sd * (float)((int)((wd >> (q * F2)) & ((1u << F2) - 1)) - (1 << (F2 - 1)));
#pragma unroll
            for (int t = 0; t < TM; ++t)
              if (t < T) acc[q][t] = fmaf(hv[t], d, acc[q][t]);
          }
        }
      }
    }
    __syncthreads();  // the wave buffer and h are reused
  }
  if (s_abort) cp_async_wait_all();

  // block rows -> yacc
#pragma unroll
  for (int t = 0; t < TM; ++t) {
    if (t < T) {
      float* dst = p.yacc + (size_t)t * H + r0;
      if (RPL >= 4) {
#pragma unroll
        for (int q = 0; q < 8; q += 4)
          if (q < RPL)
            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst + q), "f"(acc[q][t]),
                         "f"(acc[q + 1][t]), "f"(acc[q + 2][t]), "f"(acc[q + 3][t])
                         : "memory");
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (q < RPL) atomicAdd(dst + q, acc[q][t]);
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    if (s_abort) atomicAdd(p.ticket + 1, 1);
    s_last = atomic_add_acq_rel_gpu(p.ticket, 1) == (int)gridDim.x - 1;
    if (s_last && *reinterpret_cast<volatile int*>(p.ticket + 1) != 0) s_last = 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int i = tid; i < T * H; i += kChanThreads) p.y[i] = __bfloat16_as_ushort(__float2bfloat16_rn(__ldcg(p.yacc + i)));
}

}  // namespace qmoe
