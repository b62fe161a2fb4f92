// Routing, grouped-path row gather, combine and dequant kernels.
#pragma once
#include <cfloat>
#include <climits>

#include "device_common.cuh"
#include "qmm_grouped.cuh"
#include "qmm_small.cuh"
#include "unpack.cuh"

namespace qmoe {

struct RouteOut {
  int* ids;          // [T*k]
  float* w;          // [T*k]
  int* perm;         // [T*k] position -> flat index
  int* inv;          // [T*k] flat index -> position (may be null)
  int* offsets;      // [E+1]
  int* slot_token;   // [T*(k+n_shared)] (may be null)
  int* nseg;         // segment count (may be null: no segment table)
  Seg* segs;
  int max_seg;
  int* tickets;      // zeroed (may be null)
  int n_tickets;
  int thresh;        // experts with more tokens than this go to the grouped path
  int* ngseg;        // grouped tile count (may be null: no grouped table)
  GSeg* gsegs;
  int max_gseg;
  unsigned* status;
  int* chunk_counts; // [nchunks][E] (two-kernel routing)
};

// Routing of a decode batch (T <= kDecMaxT, T*k <= kDecMaxTK) as a
// standalone launch: the in-kernel routing of the decode layer kernel
// (decode_route), written out as ids, weights, the expert-sorted permutation
// and the expert offsets.  One CTA of kDecMaxT warps.
__global__ void __launch_bounds__(kDecMaxT * 32)
    route_decode_kernel(const float* __restrict__ logits, int T, int E, int k, int* ids, float* w, int* perm,
                        int* offsets) {
  __shared__ DecodeRoute R;
  decode_route(logits, T, E, k, R);
  const int TK = T * k;
  for (int i = threadIdx.x; i < TK; i += blockDim.x) {
    ids[i] = R.ids[i];
    w[i] = R.w[i];
    perm[R.pos[i]] = i;
  }
  // offsets[e]: entries routed to experts below e (segments are in expert order)
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {
    int before = 0;
    for (int r = 0; r < R.nseg; ++r)
      if (R.segs[r].expert < e) before += R.segs[r].m;
    offsets[e] = before;
  }
}

// ---- Two-kernel routing of the general path (any T) ------------------------
// route_topk_kernel: one CTA per chunk of kRouteChunk tokens; warp top-k per
// token (ties to the lower expert index), softmax over the k selected logits,
// and the chunk's per-expert counts.  route_scatter_kernel: one CTA per chunk;
// expert offsets from all chunks' counts, the chunk's base per expert from the
// chunks before it, then a stable scatter of its flat entries t*k+s in flat
// order (ranks from warp match masks and warp counts in warp order).  CTA 0
// also writes the offsets, the shared-expert slots and the segment tables.
// Deterministic: no result depends on atomics' order.
constexpr int kRouteChunk = 64;
constexpr int kRouteWarps = 8;

__device__ __forceinline__ void warp_topk(const float* __restrict__ row, int E, int k, int lane, float* selv,
                                          int* ids_out) {
  float v[kMaxExperts / 32];
  unsigned taken = 0;
  const int nv = (E + 31) >> 5;
#pragma unroll
  for (int j = 0; j < kMaxExperts / 32; ++j) {
    const int idx = lane + 32 * j;
    v[j] = (j < nv && idx < E) ? row[idx] : -FLT_MAX;
  }
  for (int s = 0; s < k; ++s) {
    float bv = -FLT_MAX;
    int bi = INT_MAX;
#pragma unroll
    for (int j = 0; j < kMaxExperts / 32; ++j) {
      const int idx = lane + 32 * j;
      if (j < nv && idx < E && !((taken >> j) & 1u) && (bi == INT_MAX || v[j] > bv)) { bv = v[j]; bi = idx; }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (oi != INT_MAX && (bi == INT_MAX || ov > bv || (ov == bv && oi < bi))) { bv = ov; bi = oi; }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == 0) {
      ids_out[s] = bi;
      selv[s] = bv;
    }
  }
  __syncwarp();
}

__global__ void __launch_bounds__(kRouteWarps * 32)
    route_topk_kernel(const float* __restrict__ logits, int T, int E, int k, RouteOut o) {
  __shared__ int cnt[kMaxExperts];
  __shared__ int sid[kRouteWarps][32];
  __shared__ float selv[kRouteWarps][32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Writes below may alias buffers the previous launch still reads.
  pdl_wait();
  pdl_trigger();
  const int t0 = blockIdx.x * kRouteChunk, t1 = min(T, t0 + kRouteChunk);
  for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int t = t0 + warp; t < t1; t += kRouteWarps) {
    warp_topk(logits + (size_t)t * E, E, k, lane, selv[warp], sid[warp]);
    if (lane < k) {
      const float lmax = selv[warp][0];
      float sum = 0.f;
      for (int s = 0; s < k; ++s) sum += expf(selv[warp][s] - lmax);
      o.w[(size_t)t * k + lane] = expf(selv[warp][lane] - lmax) / sum;
      o.ids[(size_t)t * k + lane] = sid[warp][lane];
      atomicAdd(&cnt[sid[warp][lane]], 1);  // order-independent count
    }
    __syncwarp();
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) o.chunk_counts[(size_t)blockIdx.x * E + e] = cnt[e];
}

__global__ void __launch_bounds__(kRouteWarps * 32)
    route_scatter_kernel(int T, int E, int k, int n_shared, RouteOut o) {
  __shared__ int base[kMaxExperts];   // this chunk's first position per expert (running)
  __shared__ int tot[kMaxExperts];    // all chunks' count per expert
  __shared__ int offs[kMaxExperts + 1];
  __shared__ int wtot[kRouteWarps];
  __shared__ int wcnt[kRouteWarps][kMaxExperts];
  __shared__ int seg_base[kMaxExperts + 64];
  __shared__ int gseg_base[kMaxExperts + 64];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();
  pdl_trigger();
  const int chunk = blockIdx.x, nchunks = gridDim.x;
  for (int e = tid; e < E; e += blockDim.x) {
    int before = 0, all = 0;
    for (int c = 0; c < nchunks; ++c) {
      const int v = o.chunk_counts[(size_t)c * E + e];
      all += v;
      before += c < chunk ? v : 0;
    }
    tot[e] = all;
    base[e] = before;
  }
  __syncthreads();
  // exclusive scan of tot over experts (E <= 256 = blockDim.x)
  {
    const int v = tid < E ? tot[tid] : 0;
    int inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += u;
    }
    if (lane == 31) wtot[warp] = inc;
    __syncthreads();
    int pre = 0;
    for (int w = 0; w < warp; ++w) pre += wtot[w];
    if (tid < E) {
      offs[tid] = pre + inc - v;
      base[tid] += pre + inc - v;
    }
    if (tid == E - 1) offs[E] = pre + inc;
  }
  __syncthreads();
  if (chunk == 0)
    for (int e = tid; e <= E; e += blockDim.x) o.offsets[e] = offs[e];
  // stable scatter of flat entries [i0, i1) of this chunk, in rounds of blockDim entries
  const int TK = T * k;
  const int i0 = chunk * kRouteChunk * k, i1 = min(T, (chunk + 1) * kRouteChunk) * k;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int r0 = i0; r0 < i1; r0 += blockDim.x) {
    for (int j = tid; j < kRouteWarps * kMaxExperts; j += blockDim.x) (&wcnt[0][0])[j] = 0;
    __syncthreads();
    const int i = r0 + tid;
    const bool valid = i < i1;
    const int e = valid ? o.ids[i] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & lt_mask);
    if (valid && rank == 0) wcnt[warp][e] = __popc(peers);
    __syncthreads();
    if (valid) {
      int pre = base[e];
      for (int w = 0; w < warp; ++w) pre += wcnt[w][e];
      const int pos = pre + rank;
      o.perm[pos] = i;
      if (o.inv) o.inv[i] = pos;
      if (o.slot_token) o.slot_token[pos] = i / k;
    }
    __syncthreads();
    for (int ee = tid; ee < E; ee += blockDim.x) {
      int sum = 0;
      for (int w = 0; w < kRouteWarps; ++w) sum += wcnt[w][ee];
      base[ee] += sum;
    }
    __syncthreads();
  }
  if (chunk != 0) return;
  if (o.slot_token)
    for (int i = tid; i < n_shared * T; i += blockDim.x) o.slot_token[TK + i] = i % T;
  // ---- segment tables: small-M chunks of <= 16 tokens, grouped tiles of <= 256 ----
  if (o.nseg) {
    const int EX = E + n_shared;
    if (tid == 0) {
      int sb = 0, gb = 0;
      for (int e = 0; e < EX; ++e) {
        const int cnt = e < E ? tot[e] : T;
        const bool grouped = o.ngseg && cnt > o.thresh;
        seg_base[e] = sb;
        gseg_base[e] = gb;
        if (grouped) gb += (cnt + kGTok - 1) / kGTok;
        else sb += (cnt + kChunkTokens - 1) / kChunkTokens;
      }
      if (sb > o.max_seg || (o.ngseg && gb > o.max_gseg)) {
        atomicOr(o.status, kStatusBadSegment);
        sb = 0;  // never index past the tables
        gb = 0;
      }
      *o.nseg = sb;
      if (o.ngseg) *o.ngseg = gb;
      wtot[0] = sb > 0 || gb > 0;
    }
    __syncthreads();
    const bool ok = wtot[0] != 0;
    for (int e = tid; e < EX && ok; e += blockDim.x) {
      const int cnt = e < E ? tot[e] : T;
      const int slot_base = e < E ? offs[e] : TK + (e - E) * T;
      if (o.ngseg && cnt > o.thresh) {
        const int nch = (cnt + kGTok - 1) / kGTok;
        for (int c = 0; c < nch; ++c) {
          GSeg g;
          g.expert = e;
          g.slot0 = slot_base + kGTok * c;
          g.ntok = min(kGTok, cnt - kGTok * c);
          g.pad = 0;
          o.gsegs[gseg_base[e] + c] = g;
        }
        continue;
      }
      const int nch = (cnt + kChunkTokens - 1) / kChunkTokens;
      for (int c = 0; c < nch; ++c) {
        Seg sg;
        sg.expert = e;
        sg.m = min(kChunkTokens, cnt - kChunkTokens * c);
        sg.tg = (sg.m + 7) / 8;
        sg.slot0 = slot_base + kChunkTokens * c;
        o.segs[seg_base[e] + c] = sg;
      }
    }
  }
}

// Token rows of the grouped tiles, in expert-sorted slot order: xrows[slot] =
// x[token(slot)].  One warp per row (grid-stride over gseg x 256 row slots):
// each lane moves K/256 16-byte pieces with its loads issued before its stores.
__global__ void gather_rows_kernel(const uint16_t* __restrict__ x, int K, const int* __restrict__ slot_token,
                                   const int* __restrict__ ngseg, const GSeg* __restrict__ gsegs, uint16_t* xrows) {
  pdl_wait();
  pdl_trigger();
  const int ng = *ngseg;
  const int vec = K / 8;  // uint4 per row
  const int lane = threadIdx.x & 31;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < (long long)ng * kGTok; w += nw) {
    const GSeg g = gsegs[w / kGTok];
    const int r = (int)(w % kGTok);
    if (r >= g.ntok) continue;
    const int slot = g.slot0 + r;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)slot_token[slot] * K);
    uint4* dst = reinterpret_cast<uint4*>(xrows + (size_t)slot * K);
    constexpr int kU = 8;
    for (int c0 = 0; c0 < vec; c0 += 32 * kU) {
      uint4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < vec) v[u] = __ldg(src + c);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < vec) dst[c] = v[u];
      }
    }
  }
}

// y[t] = sum_s w[t,s] * yslot[inv[t*k+s]] + sum_j yslot[T*k + j*T + t], fixed order, bf16 out.
// The token's slot indices and weights are staged in shared memory; slot rows
// are read 4 at a time so that the loads overlap.
__global__ void combine_kernel(const float* __restrict__ yslot, const float* __restrict__ w,
                               const int* __restrict__ inv, int T, int k, int n_shared, int H,
                               uint16_t* __restrict__ y) {
  __shared__ int s_row[32 + 64];
  __shared__ float s_w[32];
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  for (int i = threadIdx.x; i < k + n_shared; i += blockDim.x) {
    s_row[i] = i < k ? inv[(size_t)t * k + i] : T * k + (i - k) * T + t;
    if (i < k) s_w[i] = w[(size_t)t * k + i];
  }
  __syncthreads();
  const int ns = k + n_shared;
  for (int h = threadIdx.x * 4; h < H; h += blockDim.x * 4) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < ns; s0 += 4) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (s0 + u < ns) v[u] = *reinterpret_cast<const float4*>(yslot + (size_t)s_row[s0 + u] * H + h);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int s = s0 + u;
        if (s >= ns) break;
        if (s < k) {
          const float ws = s_w[s];
          acc.x = fmaf(ws, v[u].x, acc.x); acc.y = fmaf(ws, v[u].y, acc.y);
          acc.z = fmaf(ws, v[u].z, acc.z); acc.w = fmaf(ws, v[u].w, acc.w);
        } else {
          acc.x += v[u].x; acc.y += v[u].y; acc.z += v[u].z; acc.w += v[u].w;
        }
      }
    }
    uint2 out;
    out.x = pack_bf16x2(acc.x, acc.y);
    out.y = pack_bf16x2(acc.z, acc.w);
    *reinterpret_cast<uint2*>(y + (size_t)t * H + h) = out;
  }
}

// Clears an fp32 accumulator and a ticket array for the launch after it:
// lets that launch start at once (it waits for this one before touching
// either), then waits for the launch before, which may still use them.
__global__ void accum_reset_kernel(float* acc, int n4, int* tickets, int nt) {
  pdl_trigger();
  pdl_wait();
  const int stride = gridDim.x * blockDim.x;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride)
    reinterpret_cast<float4*>(acc)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nt; i += stride) tickets[i] = 0;
}

// Dequantize through the hot kernels' unpack: one warp per (matrix, k-unit, tile).
// Affine codes (zeros != NULL): w = s*u + z, fp32 by one fused multiply-add,
// bf16 by one bf16 fused multiply-add (a single rounding of the exact value).
template <int FMT>
__global__ void dequant_kernel(const uint8_t* __restrict__ codes, unsigned long long cstride,
                               const uint8_t* __restrict__ scales, const uint8_t* __restrict__ zeros,
                               unsigned long long sstride, int NT, int K, int block, int row_order, int nmat,
                               float* o32, uint16_t* o16) {
  using Tr = FmtTraits<FMT>;
  __shared__ uint32_t lut[243];
  if constexpr (FMT == 3)
    for (int i = threadIdx.x; i < 243; i += blockDim.x) lut[i] = tern_lut_entry(i);
  __syncthreads();
  const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const int KU = K / Tr::kKUcols;
  const long long items = (long long)nmat * KU * NT;
  const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwt = ((long long)gridDim.x * blockDim.x) >> 5;
  const int bias = FMT == 3 ? 1 : zeros ? 0 : (1 << (FMT - 1));  // code = stored field - bias
  const int rows = NT * 16;
  for (long long itm = wid; itm < items; itm += nwt) {
    const int e = (int)(itm / ((long long)KU * NT));
    const int r = (int)(itm % ((long long)KU * NT));
    const int ku = r / NT, t = r % NT;
    const uint8_t* cp = codes + (unsigned long long)e * cstride + ((unsigned long long)ku * NT + t) * Tr::kCodeBytes;
    constexpr int NKS = Tr::kKUcols / 16;
    // lane word w of this (k-unit, tile): [ku][tile][lane][W] (PLAIN, GATE_UP) or [ku][W][tile][lane] (KSPLIT)
    constexpr int W = FMT == 2 ? 2 : 4;
    auto word = [&](int w) -> uint32_t {
      if (row_order == 2)
        return *reinterpret_cast<const uint32_t*>(
            codes + (unsigned long long)e * cstride + ((((unsigned long long)ku * W + w) * NT + t) * 32 + lane) * 4);
      return *reinterpret_cast<const uint32_t*>(cp + (lane * W + w) * 4);
    };
    uint32_t am[NKS][4];
    if constexpr (FMT == 2) {
      uint32_t (&a0)[4] = am[0]; uint32_t (&a1)[4] = am[1];
      uint32_t (&a2)[4] = am[2 % NKS]; uint32_t (&a3)[4] = am[3 % NKS];
      unpack_int2_word(word(0), a0, a1);
      unpack_int2_word(word(1), a2, a3);
    } else if constexpr (FMT == 4) {
      unpack_int4_word(word(0), am[0]);
      unpack_int4_word(word(1), am[1 % NKS]);
      unpack_int4_word(word(2), am[2 % NKS]);
      unpack_int4_word(word(3), am[3 % NKS]);
    } else {
      uint8_t rec[13];
      for (int i = 0; i < 13; ++i) rec[i] = cp[lane * 13 + i];
      uint32_t ta[8][4];
      unpack_tern_record(rec, lut, ta);
#pragma unroll
      for (int ks = 0; ks < NKS; ++ks)
#pragma unroll
        for (int f = 0; f < 4; ++f) am[ks][f] = ta[ks % 8][f];
    }
    const uint8_t* sp = scales + (unsigned long long)e * sstride;
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks)
#pragma unroll
      for (int f = 0; f < 4; ++f)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float raw = h ? bf16_hi(am[ks][f]) : bf16_lo(am[ks][f]);
          const float beta = (f >= 2) ? (float)Tr::kBetaHi : 1.0f;
          const float c = (raw - 128.0f) / beta - (float)bias;
          const int pr = g + 8 * (f & 1);
          const int k = ku * Tr::kKUcols + 16 * ks + 2 * q + 8 * (f >> 1) + h;
          const size_t so = (((size_t)(k / block) * NT + t) * 8 + (pr & 7)) * 4;
          const uint32_t sw = *reinterpret_cast<const uint32_t*>(sp + so);
          const float s = pr < 8 ? bf16_lo(sw) : bf16_hi(sw);
          const int lr = row_order == 1 ? 16 * t + (pr < 8 ? 2 * pr : 2 * (pr - 8) + 1) : 16 * t + pr;
          const size_t o = ((size_t)e * rows + lr) * K + k;
          if (zeros) {
            const uint32_t zw = *reinterpret_cast<const uint32_t*>(zeros + (unsigned long long)e * sstride + so);
            const float z = pr < 8 ? bf16_lo(zw) : bf16_hi(zw);
            if (o32) o32[o] = fmaf(c, s, z);
            if (o16)
              o16[o] = __bfloat16_as_ushort(__hfma(__float2bfloat16_rn(c), __float2bfloat16_rn(s), __float2bfloat16_rn(z)));
          } else {
            const float val = c * s;
            if (o32) o32[o] = val;
            if (o16) o16[o] = __bfloat16_as_ushort(__float2bfloat16_rn(val));
          }
        }
  }
}

}  // namespace qmoe
