// Micro-benchmark: HBM read ceiling (LDG.128 and cp.async.bulk pipelines), mma.sync bf16
// throughput, and an INT2 unpack+mma mix. Standalone; all waits bounded.
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#define CK(x) do { cudaError_t e = (x); if (e != cudaSuccess) { printf("CUDA %s @%d: %s\n", #x, __LINE__, cudaGetErrorString(e)); return 1; } } while (0)

__device__ int g_err;

__global__ void read_ldg(const uint4* __restrict__ p, size_t n, unsigned long long* out) {
  uint32_t acc = 0;
  size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n; i += 4 * stride) {
    uint4 a = __ldcs(p + i), b = __ldcs(p + i + stride), c = __ldcs(p + i + 2 * stride), d = __ldcs(p + i + 3 * stride);
    acc ^= a.x ^ b.y ^ c.z ^ d.w;
  }
  for (; i < n; i += stride) { uint4 a = __ldcs(p + i); acc ^= a.x; }
  if (acc == 0x12345678u) atomicAdd(out, 1ull);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(uint64_t* b, int cnt) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(b)), "r"(cnt));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(smem_u32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t par) {
  uint32_t ok;
  asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
               : "=r"(ok) : "r"(smem_u32(b)), "r"(par) : "memory");
  return ok;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t par) {
  uint64_t t0; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (uint32_t it = 0; it < (1u << 24); ++it) {
    if (mbar_try(b, par)) return true;
    if ((it & 255) == 255) { uint64_t t1; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t1)); if (t1 - t0 > 1000000000ull) break; }
  }
  atomicExch(&g_err, 1);
  return false;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// Each warp runs its own pipeline of NST stages of CH bytes over a contiguous slice.
template <int NST, int CH>
__global__ void read_bulk(const uint8_t* __restrict__ p, size_t bytes_per_warp, unsigned long long* out) {
  extern __shared__ __align__(128) uint8_t sm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm);
  uint8_t* buf = sm + 1024 + (size_t)warp * NST * CH;
  uint64_t* wb = bars + warp * NST;
  const uint8_t* src = p + ((size_t)blockIdx.x * nw + warp) * bytes_per_warp;
  const int nch = (int)(bytes_per_warp / CH);
  if (lane == 0) for (int s = 0; s < NST; ++s) mbar_init(&wb[s], 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  __syncwarp();
  if (lane == 0)
    for (int s = 0; s < NST && s < nch; ++s) { mbar_expect_tx(&wb[s], CH); bulk_g2s(buf + s * CH, src + (size_t)s * CH, CH, &wb[s]); }
  uint32_t acc = 0;
  for (int c = 0; c < nch; ++c) {
    int s = c % NST; uint32_t par = (c / NST) & 1;
    if (!mbar_wait(&wb[s], par)) break;
    const uint32_t* w = reinterpret_cast<const uint32_t*>(buf + s * CH);
    for (int j = lane; j < CH / 4; j += 32 * 8) acc ^= w[j];
    __syncwarp();
    if (lane == 0 && c + NST < nch) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_expect_tx(&wb[s], CH); bulk_g2s(buf + s * CH, src + (size_t)(c + NST) * CH, CH, &wb[s]);
    }
  }
  if (acc == 0x12345678u) atomicAdd(out, 1ull);
}

__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, const uint32_t* b) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__global__ void mma_tput(float* out, int iters) {
  uint32_t a[4], b[2];
  for (int i = 0; i < 4; ++i) a[i] = 0x3f803f80u ^ (threadIdx.x * (i + 1));
  b[0] = 0x3f803f80u; b[1] = 0x3f80bf80u ^ threadIdx.x;
  float c[8][4] = {};
  for (int it = 0; it < iters; ++it)
#pragma unroll
    for (int j = 0; j < 8; ++j) mma16816(c[j], a, b);
  float s = 0;
  for (int j = 0; j < 8; ++j) s += c[j][0] + c[j][1] + c[j][2] + c[j][3];
  if (s == 1234.5f) out[threadIdx.x] = s;
}

__device__ __forceinline__ uint32_t lop_or(uint32_t x, uint32_t m, uint32_t magic) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(m), "r"(magic));  // (x & m) | magic
  return r;
}
__device__ __forceinline__ uint32_t hfma2_bf16(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// INT2 unpack (16 codes/u32 -> 8 bf16x2) + 2 mma per word, NTG token groups.
template <int NTG, bool NORM>
__global__ void unpack_mma(const uint32_t* __restrict__ codes, float* out, int iters) {
  uint32_t w = codes[threadIdx.x & 63];
  uint32_t b[NTG][2];
  for (int t = 0; t < NTG; ++t) { b[t][0] = 0x3f803f80u ^ t; b[t][1] = 0x3f80bf80u; }
  float c[NTG][4] = {};
  const uint32_t M = 0x43004300u;
  for (int it = 0; it < iters; ++it) {
    uint32_t w6 = w >> 6, w12 = w >> 12;
    uint32_t r[8];
    r[0] = lop_or(w, 0x00030003u, M); r[1] = lop_or(w, 0x000C000Cu, M); r[2] = lop_or(w, 0x00300030u, M);
    r[3] = lop_or(w6, 0x00030003u, M); r[4] = lop_or(w6, 0x000C000Cu, M); r[5] = lop_or(w6, 0x00300030u, M);
    r[6] = lop_or(w12, 0x00030003u, M); r[7] = lop_or(w12, 0x000C000Cu, M);
    if (NORM) {
      r[0] = hfma2_bf16(r[0], 0x3f803f80u, 0xC302C302u); r[1] = hfma2_bf16(r[1], 0x3e803e80u, 0xC208C208u);
      r[2] = hfma2_bf16(r[2], 0x3d803d80u, 0xC120C120u); r[3] = hfma2_bf16(r[3], 0x3f803f80u, 0xC302C302u);
      r[4] = hfma2_bf16(r[4], 0x3e803e80u, 0xC208C208u); r[5] = hfma2_bf16(r[5], 0x3d803d80u, 0xC120C120u);
      r[6] = hfma2_bf16(r[6], 0x3f803f80u, 0xC302C302u); r[7] = hfma2_bf16(r[7], 0x3e803e80u, 0xC208C208u);
    }
#pragma unroll
    for (int t = 0; t < NTG; ++t) { mma16816(c[t], r, b[t]); mma16816(c[t], r + 4, b[t]); }
    w = w * 1664525u + 1013904223u;
  }
  float s = 0;
  for (int t = 0; t < NTG; ++t) s += c[t][0] + c[t][1] + c[t][2] + c[t][3];
  if (s == 1234.5f) out[threadIdx.x] = s;
}

int main() {
  int dev = 0; CK(cudaSetDevice(dev));
  cudaDeviceProp pr; CK(cudaGetDeviceProperties(&pr, dev));
  int l2 = 0; CK(cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev));
  printf("dev %s SMs %d L2 %d MB smemOptin %zu\n", pr.name, pr.multiProcessorCount, l2 >> 20, pr.sharedMemPerBlockOptin);
  const int nsm = pr.multiProcessorCount;
  size_t bytes = (size_t)4 << 30;
  uint8_t* buf; CK(cudaMalloc(&buf, bytes)); CK(cudaMemset(buf, 1, bytes));
  unsigned long long* dout; CK(cudaMalloc(&dout, 64));
  float* fout; CK(cudaMalloc(&fout, 4096));
  cudaEvent_t e0, e1; cudaEventCreate(&e0); cudaEventCreate(&e1);
  float ms;
  for (int bs : {256, 512, 1024}) for (int gm : {1, 2, 4}) {
    size_t n = bytes / 16;
    read_ldg<<<nsm * gm, bs>>>((const uint4*)buf, n, dout);
    CK(cudaEventRecord(e0));
    for (int r = 0; r < 5; ++r) read_ldg<<<nsm * gm, bs>>>((const uint4*)buf, n, dout);
    CK(cudaEventRecord(e1)); CK(cudaEventSynchronize(e1)); cudaEventElapsedTime(&ms, e0, e1);
    printf("ldg bs=%d grid=%dxSM: %.1f GB/s\n", bs, gm, 5.0 * bytes / (ms * 1e6));
  }
#define RUNBULK(NST, CH, NW)                                                                  \
  {                                                                                           \
    size_t smem = 1024 + (size_t)NW * NST * CH;                                               \
    CK(cudaFuncSetAttribute(read_bulk<NST, CH>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)); \
    size_t per_warp = bytes / ((size_t)nsm * NW); per_warp -= per_warp % CH;                  \
    read_bulk<NST, CH><<<nsm, NW * 32, smem>>>(buf, per_warp, dout);                          \
    CK(cudaGetLastError());                                                                   \
    CK(cudaEventRecord(e0));                                                                  \
    for (int r = 0; r < 5; ++r) read_bulk<NST, CH><<<nsm, NW * 32, smem>>>(buf, per_warp, dout); \
    CK(cudaEventRecord(e1)); CK(cudaEventSynchronize(e1)); cudaEventElapsedTime(&ms, e0, e1);  \
    printf("bulk nst=%d ch=%d warps=%d inflight/SM=%zuKB: %.1f GB/s\n", NST, CH, NW, (size_t)NW * NST * CH / 1024, \
           5.0 * per_warp * nsm * NW / (ms * 1e6));                                           \
  }
  RUNBULK(4, 4096, 8) RUNBULK(3, 4096, 8) RUNBULK(3, 8192, 8) RUNBULK(6, 4096, 8) RUNBULK(4, 2048, 16) RUNBULK(2, 8192, 8)
  RUNBULK(4, 16384, 2) RUNBULK(3, 16384, 4) RUNBULK(4, 8192, 4)
  int h_err = 0; CK(cudaMemcpyFromSymbol(&h_err, g_err, sizeof(int))); printf("bulk wait errors: %d\n", h_err);

  for (int warps : {4, 8, 16}) {
    int iters = 4096;
    mma_tput<<<nsm, warps * 32>>>(fout, 16);
    CK(cudaEventRecord(e0)); mma_tput<<<nsm, warps * 32>>>(fout, iters); CK(cudaEventRecord(e1));
    CK(cudaEventSynchronize(e1)); cudaEventElapsedTime(&ms, e0, e1);
    double fl = 2.0 * 16 * 8 * 16 * 8.0 * iters * warps * nsm;
    printf("mma.sync m16n8k16 bf16 warps/SM=%d: %.1f TFLOP/s\n", warps, fl / (ms * 1e9));
  }
  uint32_t* codes; CK(cudaMalloc(&codes, 4096)); CK(cudaMemset(codes, 0x5a, 4096));
#define RUNUM(NTG, NORM, WARPS)                                                              \
  {                                                                                          \
    int iters = 4096;                                                                        \
    unpack_mma<NTG, NORM><<<nsm, WARPS * 32>>>(codes, fout, 16);                              \
    CK(cudaEventRecord(e0)); unpack_mma<NTG, NORM><<<nsm, WARPS * 32>>>(codes, fout, iters); CK(cudaEventRecord(e1)); \
    CK(cudaEventSynchronize(e1)); cudaEventElapsedTime(&ms, e0, e1);                           \
    double wts = 16.0 * 32 * iters * WARPS * nsm;                                            \
    printf("int2 unpack+mma ntg=%d norm=%d warps=%d: %.2f Tweights/s (= %.0f GB/s of INT2 codes)\n", NTG, NORM, WARPS, \
           wts / (ms * 1e9), wts / 4 / (ms * 1e6));                                          \
  }
  RUNUM(1, true, 8) RUNUM(1, false, 8) RUNUM(1, true, 16) RUNUM(2, true, 8) RUNUM(4, true, 8) RUNUM(1, true, 32)
  CK(cudaDeviceSynchronize());
  printf("done\n");
  return 0;
}
