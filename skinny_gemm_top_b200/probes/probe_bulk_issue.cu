// Probe: issue cost of cp.async.bulk when L lanes of one warp issue concurrently (148 CTAs, 1 warp each).
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
#define CK(x) do { cudaError_t e = (x); if (e != cudaSuccess) { printf("CUDA %s: %s\n", #x, cudaGetErrorString(e)); return 1; } } while (0)
__device__ __forceinline__ uint32_t sa(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ unsigned long long gt() { unsigned long long t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t)); return t; }
__device__ __forceinline__ long long clk() { long long c; asm volatile("mov.u64 %0, %%clock64;" : "=l"(c) :: "memory"); return c; }
__global__ void issue(const uint8_t* src, int bytes, int total, int lanes, long long* out) {
  extern __shared__ __align__(128) uint8_t sm[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm);
  uint8_t* buf = sm + 128;
  const int lane = threadIdx.x;
  if (lane == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" :: "r"(sa(bar)));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(sa(bar)), "r"(bytes * total) : "memory");
  }
  __syncwarp();
  const uint8_t* g = src + (size_t)blockIdx.x * total * bytes;
  long long c0 = clk();
  if (lane < lanes)
    for (int i = lane; i < total; i += lanes)
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                   :: "r"(sa(buf + (size_t)i * bytes)), "l"(g + (size_t)i * bytes), "r"(bytes), "r"(sa(bar)) : "memory");
  __syncwarp();
  long long c1 = clk();
  uint32_t ok = 0;
  unsigned long long t0 = gt();
  if (lane == 0)
    while (!ok) {
      asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0; selp.u32 %0,1,0,p; }" : "=r"(ok) : "r"(sa(bar)) : "memory");
      if (gt() - t0 > 1000000000ull) break;
    }
  __syncwarp();
  long long c2 = clk();
  if (lane == 0) { out[blockIdx.x * 3] = c1 - c0; out[blockIdx.x * 3 + 1] = c2 - c0; out[blockIdx.x * 3 + 2] = ok; }
}
int main() {
  uint8_t* src; CK(cudaMalloc(&src, (size_t)1 << 30)); CK(cudaMemset(src, 1, (size_t)1 << 30));
  long long* dout; CK(cudaMalloc(&dout, 148 * 3 * 8));
  long long h[148 * 3];
  CK(cudaFuncSetAttribute(issue, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024));
  for (int bytes : {256, 1024, 4096})
    for (int lanes : {1, 4, 8, 32}) {
      const int total = bytes == 4096 ? 32 : (bytes == 1024 ? 64 : 128);
      for (int rep = 0; rep < 3; ++rep) { issue<<<148, 32, 128 + total * bytes>>>(src, bytes, total, lanes, dout); CK(cudaDeviceSynchronize()); }
      CK(cudaMemcpy(h, dout, sizeof(h), cudaMemcpyDeviceToHost));
      double iss = 0, all = 0; int okc = 0;
      for (int b = 0; b < 148; ++b) { iss += h[3 * b]; all += h[3 * b + 1]; okc += (int)h[3 * b + 2]; }
      printf("bytes %5d copies %3d lanes %2d: issue %7.0f cycles (%.1f per copy), to completion %7.0f cycles, ok %d\n",
             bytes, total, lanes, iss / 148, iss / 148 / total, all / 148, okc);
    }
  printf("done\n");
  return 0;
}
