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
// Launches, chained by programmatic dependent launch (after a reset of the
// histogram, the accumulator and the tickets):
//   chan_score_kernel   routing, rotation of x, sketch products, scores and a
//                       histogram of their top bits
//   chan_select_kernel  one block per token: radix select of the n_keep best
//   chan_exact_kernel   the selected and shared channel records: gate/up dot
//                       products, SwiGLU, down-column accumulation, combine
//
// A channel (and its sketch) is one contiguous record, so a block's work is a
// list of records streamed into shared memory with 16-byte cp.async by every
// thread, completing on mbarriers (a few per wave).  The dot products run on
// the CUDA cores: a code u is turned into the float 1 + u / 2^bits (one shift
// and one LOP3 into the mantissa), multiplied with x, and the constant part is
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
constexpr int kSelThreads = 256;
constexpr int kChanMaxCand = 32768;  // k * I of one token (selection block's shared memory)
constexpr int kSketchBlock = 128;
constexpr int kChanBins = 4096;  // first selection level: score bits 30..19
constexpr int kChanChunks = 4;   // copy barriers per wave of the score kernel
constexpr int kChanMaxH = 2048;  // FC2 of the exact kernel: 16 warps x 128 output rows

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
  int* hist;              // [T][kChanBins] counts of the scores' top bits, zeroed before the score kernel
  float* yacc;            // [T][H] fp32 accumulator, zeroed before the score kernel
  int* ticket;            // [0] exact-kernel blocks done, [1] blocks that gave up
  uint16_t* y;            // [T][H] bf16
  float inv_sqrt_h;       // 1 / sqrt(H)
  int wave_sk;            // sketch records per wave of the score kernel
  int wave_rec;           // channel records per wave of the exact kernel
  unsigned long long wait_ns;
  int inject;             // test hook: 1 = every exact-kernel block waits on a barrier nothing arrives at
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

// (d0, d1) += (a0, a1) * (b0, b1): one packed fp32 FMA (two IEEE fused multiply-adds).
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rd, {%0, %1};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rd;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Balanced split of n units over the grid.
__device__ __forceinline__ void chan_range(int n, int* lo, int* hi) {
  *lo = (int)((long long)n * blockIdx.x / gridDim.x);
  *hi = (int)((long long)n * (blockIdx.x + 1) / gridDim.x);
}

// All threads: 16-byte cp.async of records [ia, ib) of `bytes` bytes each
// (sources in src[]) into their slots of buf.  The caller arrives on the wave's
// barrier (count kChanThreads) once all of its pieces are issued.
__device__ __forceinline__ void chan_copy_units(uint8_t* buf, const uint8_t* const* src, int ia, int ib,
                                                int bytes) {
  const int per = bytes >> 4;
  const int total = (ib - ia) * per;
  for (int c = threadIdx.x; c < total; c += kChanThreads) {
    const int i = ia + c / per, o = c - (i - ia) * per;
    cp_async16(buf + (size_t)i * bytes + 16 * o, src[i] + 16 * o);
  }
}

// ---------------------------------------------------------------------------
// Scores.  Units: (active expert a, channel j), a over the distinct routed
// experts of the batch in ascending id; every token routed to a gets the
// score of channel j from one read of its sketch record.  TM >= T bounds the
// tokens per expert (the per-token accumulators are registers).
//
// Shared memory: x' [T][4][H/16] float4 (word-interleaved: element c at word
// c / 16, quarter (c / 4) % 4, component c % 4), per-word sums of x' [T][H/16],
// record sources, then the wave of sketch records.

// Float offset of natural element c in the word-interleaved layout (W16 = 2^lgw words).
__device__ __forceinline__ int xq_off(int c, int lgw) {
  return (c & 3) | ((c >> 4) << 2) | (((c >> 2) & 3) << (lgw + 2));
}

// Unscaled Walsh-Hadamard transform (Sylvester order) of T rows of H = 2^lgh
// floats held in the word-interleaved layout, in place: radix-4 passes (two
// stages per barrier), then one radix-2 pass when lgh is odd.
__device__ __forceinline__ void fwht_rows(float* xs, int T, int lgh) {
  const int H = 1 << lgh, lgw = lgh - 4;
  for (int lg = 0; lg + 1 < lgh; lg += 2) {
    const int len = 1 << lg;
    for (int b = threadIdx.x; b < T * (H >> 2); b += kChanThreads) {
      const int t = b >> (lgh - 2), g = b & ((H >> 2) - 1);
      const int i0 = ((g >> lg) << (lg + 2)) | (g & (len - 1));
      float* row = xs + ((size_t)t << lgh);
      const int o0 = xq_off(i0, lgw), o1 = xq_off(i0 + len, lgw), o2 = xq_off(i0 + 2 * len, lgw),
                o3 = xq_off(i0 + 3 * len, lgw);
      const float a0 = row[o0], a1 = row[o1], a2 = row[o2], a3 = row[o3];
      const float s01 = a0 + a1, d01 = a0 - a1, s23 = a2 + a3, d23 = a2 - a3;
      row[o0] = s01 + s23;
      row[o1] = d01 + d23;
      row[o2] = s01 - s23;
      row[o3] = d01 - d23;
    }
    __syncthreads();
  }
  if (lgh & 1) {
    const int len = H >> 1;
    for (int b = threadIdx.x; b < T * len; b += kChanThreads) {
      const int t = b >> (lgh - 1), i = b & (len - 1);
      float* row = xs + ((size_t)t << lgh);
      const int o0 = xq_off(i, lgw), o1 = xq_off(i + len, lgw);
      const float a0 = row[o0], a1 = row[o1];
      row[o0] = a0 + a1;
      row[o1] = a0 - a1;
    }
    __syncthreads();
  }
}

template <int TM, int NWL>  // NWL: sketch words per lane per row (H = 512 * NWL)
__global__ void __launch_bounds__(kChanThreads, 1) chan_score_kernel(ChanParams p) {
  constexpr int H = 512 * NWL, W16 = H / 16, SKB = H / kSketchBlock, LGH = NWL == 1 ? 9 : NWL == 2 ? 10 : 11;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t bar[kChanChunks];
  __shared__ int s_ids[kChanMaxAct];
  __shared__ float s_w[kChanMaxAct];
  __shared__ int s_act_e[kChanMaxAct], s_act_n[kChanMaxAct], s_act_m[kChanMaxAct][kChanMaxT];
  __shared__ int s_nact, s_abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = p.T, I = p.I, k = p.k;
  constexpr int lgh = LGH;
  // shared memory by offsets from the array (so every access stays a shared-memory access)
  float* xs = reinterpret_cast<float*>(smem);
  float* sxw = xs + T * H;
  const int src_off = (4 * (T * H + T * W16) + 15) & ~15;
  const uint8_t** src = reinterpret_cast<const uint8_t**>(smem + src_off);
  const int buf_off = (src_off + 8 * p.wave_sk + 127) & ~127;
  uint8_t* buf = smem + buf_off;

  if (tid == 0) {
    for (int c = 0; c < kChanChunks; ++c) mbar_init(&bar[c], kChanThreads);
    fence_mbar_init();
    s_abort = 0;
  }
  pdl_wait();
  pdl_trigger();

  if (warp < T) chan_route_token(p.logits + (size_t)warp * p.E, p.E, k, lane, s_ids + warp * k, s_w + warp * k);
  // x * d into the word-interleaved layout (four independent loads per thread in flight)
  for (int i0 = tid * 4; i0 < T * H; i0 += kChanThreads * 4) {
    const int t = i0 >> lgh, c = i0 & (H - 1);
    const uint2 xv = *reinterpret_cast<const uint2*>(p.x + (size_t)t * H + c);
    const float4 sg = *reinterpret_cast<const float4*>(p.signs + c);
    float* row = xs + ((size_t)t << lgh);
    const int o = xq_off(c, lgh - 4);  // c % 4 == 0: four consecutive floats
    row[o] = bf16_lo(xv.x) * sg.x;
    row[o + 1] = bf16_hi(xv.x) * sg.y;
    row[o + 2] = bf16_lo(xv.y) * sg.z;
    row[o + 3] = bf16_hi(xv.y) * sg.w;
  }
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

  // a wave of sketch records in kChanChunks consecutive groups, one barrier each
  auto chunk_lo = [](int c, int nw) { return c * nw / kChanChunks; };
  auto issue = [&](int w0, int nw) {
    for (int i = tid; i < nw; i += kChanThreads) {
      const int u = w0 + i, a = u / I, j = u - a * I;
      src[i] = p.sketch + ((size_t)s_act_e[a] * I + j) * skb;
    }
    __syncthreads();
    for (int c = 0; c < kChanChunks; ++c) {
      chan_copy_units(buf, src, chunk_lo(c, nw), chunk_lo(c + 1, nw), skb);
      cp_async_arrive(&bar[c]);
    }
  };
  if (u0 < u1) issue(u0, min(p.wave_sk, u1 - u0));

  // x' = Had (d * x), unscaled (1/sqrt(H) is applied to the products), while the sketch lands
  fwht_rows(xs, T, lgh);
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
  int wave = 0;
  for (int w0 = u0; w0 < u1; w0 += p.wave_sk, ++wave) {
    const int nw = min(p.wave_sk, u1 - w0);
    if (w0 != u0) issue(w0, nw);
    int ready = 0;  // chunks of this wave known to have landed (per warp)
    for (int i = warp; i < nw; i += kChanWarps) {
      while (ready < kChanChunks && i >= chunk_lo(ready, nw)) {
        if (__any_sync(0xffffffffu, !mbar_wait_sleep_bounded(&bar[ready], wave & 1, p.status, p.wait_ns)))
          s_abort = 1;
        ++ready;
      }
      if (*reinterpret_cast<volatile int*>(&s_abort)) break;
      const int u = w0 + i, a = u / I, j = u - a * I;
      const int nm = s_act_n[a];
      const uint8_t* r = buf + i * p.sk_bytes;
      const uint32_t* gw = reinterpret_cast<const uint32_t*>(r) + lane;
      const uint16_t* sc = reinterpret_cast<const uint16_t*>(r + H / 2);
      int tok[TM];
#pragma unroll
      for (int m = 0; m < TM; ++m) tok[m] = m < nm ? s_act_m[a][m] / k : 0;
      float ag[TM], au[TM];
#pragma unroll
      for (int m = 0; m < TM; ++m) ag[m] = au[m] = 0.f;
#pragma unroll
      for (int n = 0; n < NWL; ++n) {
        const int w = lane + 32 * n;
        const uint32_t g = gw[32 * n], uu = gw[W16 + 32 * n];
        const float sg = bf16_to_f(sc[w >> 3]), su = bf16_to_f(sc[SKB + (w >> 3)]);
        float vg[16], vu[16];
        Unroll<16>::run([&](auto kk) {
          constexpr int K = decltype(kk)::value;
          vg[K] = code2_f<K>(g);
          vu[K] = code2_f<K>(uu);
        });
#pragma unroll
        for (int m = 0; m < TM; ++m) {
          if (TM == 1 || m < nm) {
            const int t = tok[m];
            float dg0 = 0.f, dg1 = 0.f, du0 = 0.f, du1 = 0.f;
            const float4* xr = x4 + t * 4 * W16 + w;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4 xv = xr[q * W16];
              ffma2(dg0, dg1, vg[4 * q], vg[4 * q + 1], xv.x, xv.y);
              ffma2(du0, du1, vu[4 * q], vu[4 * q + 1], xv.x, xv.y);
              ffma2(dg0, dg1, vg[4 * q + 2], vg[4 * q + 3], xv.z, xv.w);
              ffma2(du0, du1, vu[4 * q + 2], vu[4 * q + 3], xv.z, xv.w);
            }
            const float sx = 6.f * sxw[t * W16 + w];
            ag[m] = fmaf(sg, fmaf(4.f, dg0 + dg1, -sx), ag[m]);
            au[m] = fmaf(su, fmaf(4.f, du0 + du1, -sx), au[m]);
          }
        }
      }
      const int e = s_act_e[a];
      const float dnj = p.dn[(size_t)e * I + j];
#pragma unroll
      for (int m = 0; m < TM; ++m) {
        if (TM == 1 || m < nm) {
          const float gs = warp_sum(ag[m]) * p.inv_sqrt_h, us = warp_sum(au[m]) * p.inv_sqrt_h;
          if (lane == m) {
            const int mm = s_act_m[a][m], t = mm / k, s = mm - t * k;
            const float sc = s_w[mm] * dnj * fabsf(silu_f(gs) * us);
            p.scores[((size_t)t * k + s) * I + j] = sc;
            atomicAdd(p.hist + t * kChanBins + ((__float_as_uint(sc) & 0x7FFFFFFFu) >> 19), 1);
          }
        }
      }
    }
    // every chunk barrier of the wave completes before the buffer is reused
    for (; ready < kChanChunks; ++ready)
      if (!mbar_wait_sleep_bounded(&bar[ready], wave & 1, p.status, p.wait_ns)) s_abort = 1;
    __syncthreads();
    if (s_abort) break;
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

// The bin (of nb, counts in h, digit order = key order) holding the need-th
// largest key: returns it, and in *above the count of keys in higher bins.
// Each thread takes nb / kSelThreads consecutive bins, highest first.
__device__ __forceinline__ int sel_find_bin(const int* h, int nb, int need, int* above, int* sh, int* s_res) {
  const int per = nb / kSelThreads, hi = nb - 1 - per * (int)threadIdx.x;
  int tot = 0;
  for (int m = 0; m < per; ++m) tot += h[hi - m];
  int excl, unused;
  block_scan2(tot, 0, &excl, &unused, sh);
  if (excl < need && need <= excl + tot) {
    int run = excl;
    for (int m = 0; m < per; ++m) {
      if (run + h[hi - m] >= need) {
        s_res[0] = hi - m;
        s_res[1] = run;
        break;
      }
      run += h[hi - m];
    }
  }
  __syncthreads();
  const int b = s_res[0];
  *above = s_res[1];
  __syncthreads();
  return b;
}

// Selection of one token (block t): the n_keep best scores by a three-level
// radix select on the score bits (scores are >= 0, so their bit patterns
// order like the values).  Level 1 (bits 30..19) was counted by the score
// kernel; levels 2 (bits 18..7) and 3 (bits 6..0) count only the keys left in
// the boundary bin.  Then the selected indices are written in ascending order
// (ties at the threshold key to the lower index).  Keys sit in shared memory,
// each thread owning a contiguous run of them.
__global__ void __launch_bounds__(kSelThreads, 1) chan_select_kernel(ChanParams p) {
  extern __shared__ __align__(16) uint32_t keys[];
  __shared__ int hist[kChanBins];
  __shared__ int sh[64];
  __shared__ int s_res[2];
  const int tid = threadIdx.x;
  const int t = blockIdx.x, n = p.k * p.I;
  pdl_wait();
  pdl_trigger();
  if (tid == 0) s_res[0] = s_res[1] = 0;
  // scores and the level-1 histogram into shared memory, every element's copy in flight at once
  const float* sc = p.scores + (size_t)t * n;
  for (int i = tid; i < n; i += kSelThreads) cp_async4(keys + i, sc + i);
  const int* h1 = p.hist + (size_t)t * kChanBins;
  for (int i = tid; i < kChanBins / 4; i += kSelThreads) cp_async16(hist + 4 * i, h1 + 4 * i);
  cp_async_wait_all();
  __syncthreads();
  for (int i = tid; i < n; i += kSelThreads) keys[i] &= 0x7FFFFFFFu;
  __syncthreads();
  const int per = (n + kSelThreads - 1) / kSelThreads;
  const int lo = min(n, tid * per), hi = min(n, lo + per);
  int above, need = p.n_keep;
  const int b1 = sel_find_bin(hist, kChanBins, need, &above, sh, s_res);
  need -= above;
  for (int i = tid; i < kChanBins; i += kSelThreads) hist[i] = 0;
  __syncthreads();
  for (int i = lo; i < hi; ++i)  // level 2: keys of bin b1, by bits 18..7
    if ((int)(keys[i] >> 19) == b1) atomicAdd(&hist[(keys[i] >> 7) & 4095u], 1);
  __syncthreads();
  const int b2 = sel_find_bin(hist, kChanBins, need, &above, sh, s_res);
  need -= above;
  for (int i = tid; i < kChanBins; i += kSelThreads) hist[i] = 0;
  __syncthreads();
  const uint32_t pre = ((uint32_t)b1 << 19) | ((uint32_t)b2 << 7);
  for (int i = lo; i < hi; ++i)  // level 3: keys of bins (b1, b2), by bits 6..0
    if ((keys[i] & ~127u) == pre) atomicAdd(&hist[keys[i] & 127u], 1);
  __syncthreads();
  const int b3 = sel_find_bin(hist, kSelThreads, need, &above, sh, s_res);  // 128 bins, one per thread
  need = max(need - above, 0);
  const uint32_t theta = pre | (uint32_t)b3;  // key of the n_keep-th best; `need` keys equal to it are taken
  int gt = 0, eq = 0;
  for (int i = lo; i < hi; ++i) {
    gt += keys[i] > theta;
    eq += keys[i] == theta;
  }
  int gt0, eq0;
  block_scan2(gt, eq, &gt0, &eq0, sh);
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
// memory; then FC2 with warp w owning output rows [128 w, 128 w + 128) (four
// per lane) for every record of the wave, accumulated in registers; at the end
// the block's rows are added into yacc and the last block rounds y to bf16.
// H <= 2048.  TM >= T bounds the tokens (register accumulators).
//
// The shared experts' records depend on nothing the selection writes: they
// are requested before griddepcontrol.wait, together with x (which every
// kernel of the chain has seen complete by the time this one launches).
template <int F1, int F2, int TM>
__global__ void __launch_bounds__(kChanThreads, 1) chan_exact_kernel(ChanParams p) {
  constexpr int CPC = 128 / F1;  // columns per 16-byte chunk of a gate/up row
  constexpr int LCPC = F1 == 4 ? 5 : 6;
  constexpr int CPW = 32 / F1;   // columns per 32-bit word
  constexpr float kA = F1 == 4 ? 16.f : 4.f;  // sum c x = kA * sum v x - kB * sum x
  constexpr float kB = F1 == 4 ? 24.f : 6.f;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t bar[2];  // per wave: [0] its shared-expert records, [1] its selected records
  __shared__ uint64_t dbar;    // test hook: a barrier nothing arrives at
  __shared__ int s_last, s_abort;
  __shared__ int s_ids[kChanMaxAct];
  __shared__ float s_wts[kChanMaxAct];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H, T = p.T, I = p.I, NC = H >> LCPC, R = p.rec_bytes, WR = p.wave_rec;
  const int SB = H / p.block;
  const int off_u = H * F1 / 8, off_d = 2 * off_u, off_s = off_d + H * F2 / 8;
  float* xs = reinterpret_cast<float*>(smem);                       // [T][CPC/4][NC] float4
  float* sxc = xs + (size_t)T * H;                                  // [T][NC]
  float* hc = sxc + (size_t)T * NC;                                 // [WR][TM]
  int* utok = reinterpret_cast<int*>(hc + (size_t)WR * TM);         // [WR]: token, or -1 for all
  float* uw = reinterpret_cast<float*>(utok + WR);                  // [WR]: weight
  // by offsets from the array, so that every access stays a shared-memory access
  const int src_off = (4 * (T * H + T * NC + WR * TM + 2 * WR) + 15) & ~15;
  const uint8_t** src = reinterpret_cast<const uint8_t**>(smem + src_off);
  uint8_t* buf = smem + ((src_off + 8 * WR + 127) & ~127);

  if (tid == 0) {
    mbar_init(&bar[0], kChanThreads);
    mbar_init(&bar[1], kChanThreads);
    mbar_init(&dbar, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  const int n_sh = p.S * I;
  int u0, u1;
  chan_range(n_sh + T * p.n_keep, &u0, &u1);
  auto unit_shared = [&](int i, int u) {
    src[i] = p.rec + ((size_t)(p.E + u / I) * I + (u % I)) * R;
    utok[i] = -1;
    uw[i] = 1.f;
  };
  auto unit_routed = [&](int i, int u) {
    const int v = u - n_sh, t = v / p.n_keep;
    const int f = p.sel[v];
    const int s = f / I;
    int e = (f >= 0 && s < p.k) ? s_ids[t * p.k + s] : -1;
    int j = f - s * I;
    float wt = e >= 0 ? s_wts[t * p.k + s] : 0.f;
    if (e < 0 || e >= p.E) {  // a corrupt selection: read record 0, add nothing
      atomicOr(p.status, kStatusBadSegment);
      e = 0;
      j = 0;
      wt = 0.f;
    }
    src[i] = p.rec + ((size_t)e * I + j) * R;
    utok[i] = t;
    uw[i] = wt;
  };
  // routing of the score kernel: with a selection step in between, the score
  // kernel has completed before this kernel launches (every kernel of the chain
  // waits for its predecessor before it lets the next one start)
  if (p.n_keep > 0 && tid < T * p.k) {
    s_ids[tid] = p.ids[tid];
    s_wts[tid] = p.wts[tid];
  }
  // first wave's shared-expert records, before the wait
  const int nw0 = min(WR, u1 - u0), ns0 = max(0, min(nw0, n_sh - u0));
  for (int i = tid; i < ns0; i += kChanThreads) unit_shared(i, u0 + i);
  __syncthreads();
  chan_copy_units(buf, src, 0, ns0, R);
  cp_async_arrive(&bar[0]);
  // x (bf16) -> [T][CPC/4][NC] fp32, and the per-chunk sums of x
  for (int i0 = tid * 4; i0 < T * H; i0 += kChanThreads * 4) {
    const int t = i0 / H, c = i0 - t * H;
    const uint2 xv = *reinterpret_cast<const uint2*>(p.x + (size_t)t * H + c);
    const int ch = c >> LCPC, q = (c & (CPC - 1)) >> 2;
    float4* d = reinterpret_cast<float4*>(xs) + ((size_t)t * (CPC / 4) + q) * NC + ch;
    *d = make_float4(bf16_lo(xv.x), bf16_hi(xv.x), bf16_lo(xv.y), bf16_hi(xv.y));
  }
  pdl_wait();
  pdl_trigger();
  for (int i = ns0 + tid; i < nw0; i += kChanThreads) unit_routed(i, u0 + i);
  __syncthreads();
  chan_copy_units(buf, src, ns0, nw0, R);
  cp_async_arrive(&bar[1]);
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

  const int r0 = warp * 128 + lane * 4;  // FC2 rows of this lane (H <= 2048: 16 warps cover H)
  const bool has_rows = r0 < H;
  float acc[4][TM];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int t = 0; t < TM; ++t) acc[q][t] = 0.f;

  int wave = 0;
  for (int w0 = u0; w0 < u1; w0 += WR, ++wave) {
    const int nw = min(WR, u1 - w0), nsw = max(0, min(nw, n_sh - w0));  // nsw: shared records first
    if (w0 != u0) {
      for (int i = tid; i < nw; i += kChanThreads) {
        if (i < nsw) unit_shared(i, w0 + i);
        else unit_routed(i, w0 + i);
      }
      __syncthreads();
      chan_copy_units(buf, src, 0, nsw, R);
      cp_async_arrive(&bar[0]);
      chan_copy_units(buf, src, nsw, nw, R);
      cp_async_arrive(&bar[1]);
    }
    int ready = 0;  // barriers of this wave this warp has seen complete

    // FC1: one warp per record (shared records first, so the first barrier often suffices)
    for (int i = warp; i < nw; i += kChanWarps) {
      while (ready < 2 && (ready == 0 || i >= nsw)) {
        if (__any_sync(0xffffffffu, !mbar_wait_sleep_bounded(&bar[ready], wave & 1, p.status, p.wait_ns)))
          s_abort = 1;
        ++ready;
      }
      if (*reinterpret_cast<volatile int*>(&s_abort)) break;
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
        const int blk = (ch << LCPC) / p.block;
        const float sg = bf16_to_f(sc[blk]), su = bf16_to_f(sc[SB + blk]);
        const uint32_t gw[4] = {G.x, G.y, G.z, G.w}, uwd[4] = {U.x, U.y, U.z, U.w};
        float dg[TM], du[TM], dg1[TM], du1[TM];
#pragma unroll
        for (int m = 0; m < TM; ++m) dg[m] = du[m] = dg1[m] = du1[m] = 0.f;
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
            if (TM == 1 || m < nt) {
              const int t = tok < 0 ? m : tok;
#pragma unroll
              for (int qq = 0; qq < CPW / 4; ++qq) {
                const float4 xv = x4[((size_t)t * (CPC / 4) + wd * (CPW / 4) + qq) * NC + ch];
                ffma2(dg[m], dg1[m], vg[4 * qq], vg[4 * qq + 1], xv.x, xv.y);
                ffma2(du[m], du1[m], vu[4 * qq], vu[4 * qq + 1], xv.x, xv.y);
                ffma2(dg[m], dg1[m], vg[4 * qq + 2], vg[4 * qq + 3], xv.z, xv.w);
                ffma2(du[m], du1[m], vu[4 * qq + 2], vu[4 * qq + 3], xv.z, xv.w);
              }
            }
          }
        }
#pragma unroll
        for (int m = 0; m < TM; ++m) {
          if (TM == 1 || m < nt) {
            const float sx = kB * sxc[(tok < 0 ? m : tok) * NC + ch];
            ag[m] = fmaf(sg, fmaf(kA, dg[m] + dg1[m], -sx), ag[m]);
            au[m] = fmaf(su, fmaf(kA, du[m] + du1[m], -sx), au[m]);
          }
        }
      }
      const float wt = uw[i];
      if (tok < 0) {  // a shared expert: every token
#pragma unroll
        for (int m = 0; m < TM; ++m) {
          float h = 0.f;
          if (TM == 1 || m < T) h = wt * silu_f(warp_sum(ag[m])) * warp_sum(au[m]);
          if (lane == 0) hc[i * TM + m] = h;
        }
      } else {
        const float h = wt * silu_f(warp_sum(ag[0])) * warp_sum(au[0]);
        if (lane == 0)
#pragma unroll
          for (int m = 0; m < TM; ++m) hc[i * TM + m] = m == tok ? h : 0.f;
      }
    }
    for (; ready < 2; ++ready)
      if (!mbar_wait_sleep_bounded(&bar[ready], wave & 1, p.status, p.wait_ns)) s_abort = 1;
    __syncthreads();
    if (s_abort) break;

    // FC2: rows r0 .. r0 + 3 of every record of the wave
    if (has_rows) {
      const int wsh = (r0 * F2) & 31, widx = (r0 * F2) >> 5, sbl = r0 / p.block;
      for (int i = 0; i < nw; ++i) {
        const uint8_t* r = buf + (size_t)i * R;
        const uint32_t wd = reinterpret_cast<const uint32_t*>(r + off_d)[widx] >> wsh;
        const float sd = bf16_to_f(reinterpret_cast<const uint16_t*>(r + off_s)[2 * SB + sbl]);
        float hv[TM];
#pragma unroll
        for (int t = 0; t < TM; ++t) hv[t] = hc[i * TM + t];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float d = sd * (float)((int)((wd >> (q * F2)) & ((1u << F2) - 1)) - (1 << (F2 - 1)));
#pragma unroll
          for (int t = 0; t < TM; ++t) acc[q][t] = fmaf(hv[t], d, acc[q][t]);
        }
      }
    }
    __syncthreads();  // the wave buffer and h are reused
  }
  if (p.inject == 1 && tid == 0 && !mbar_wait_sleep_bounded(&dbar, 0, p.status, p.wait_ns)) s_abort = 1;
  __syncthreads();
  if (s_abort) cp_async_wait_all();

  // block rows -> yacc (a block that gave up adds nothing; the last block then leaves y as it was)
  if (has_rows && !s_abort) {
#pragma unroll
    for (int t = 0; t < TM; ++t) {
      if (TM == 1 || t < T)
        asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p.yacc + (size_t)t * H + r0),
                     "f"(acc[0][t]), "f"(acc[1][t]), "f"(acc[2][t]), "f"(acc[3][t])
                     : "memory");
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
