// Probe: streaming HBM read through per-warp SMEM stage pipelines with 1, 2 or 4 warps per CTA (148 CTAs):
// mode 0: cp.async.cg 16 B per lane + cp.async.mbarrier.arrive.noinc
// mode 1: one cp.async.bulk per stage (lane 0), expect_tx
// mode 2: bulk for (stage - 256) bytes + cp.async for the last 256 bytes
// All waits bounded (2 s of globaltimer), timeout recorded in a flag.
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
#define CK(x) do { cudaError_t e = (x); if (e != cudaSuccess) { printf("CUDA %s: %s\n", #x, cudaGetErrorString(e)); return 1; } } while (0)
__device__ __forceinline__ uint32_t sa(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ unsigned long long gt() { unsigned long long t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t)); return t; }
__device__ __forceinline__ bool try_wait(uint64_t* bar, uint32_t par) {
  uint32_t ok;
  asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0,1,0,p; }" : "=r"(ok) : "r"(sa(bar)), "r"(par) : "memory");
  return ok;
}
__device__ bool wait_b(uint64_t* bar, uint32_t par) {
  if (try_wait(bar, par)) return true;
  unsigned long long t0 = gt();
  for (uint32_t it = 1;; ++it) {
    if (try_wait(bar, par)) return true;
    if ((it & 255) == 0 && gt() - t0 > 2000000000ull) return false;
  }
}
__global__ void __launch_bounds__(256, 1) stream(const uint8_t* src, int mode, int sbytes, int nst, int items, unsigned* flag, unsigned* sink) {
  const int WPC = blockDim.x >> 5;
  extern __shared__ __align__(128) uint8_t sm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm) + warp * 16;
  uint8_t* st = sm + 2048 + (size_t)warp * nst * sbytes;
  const int cnt = mode == 0 ? 32 : (mode == 1 ? 1 : 33);
  if (lane == 0) for (int s = 0; s < nst; ++s) asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(sa(&bars[s])), "r"(cnt));
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  __syncthreads();
  // item i of warp w (global warp id gw) reads chunk (i * nwarps + gw)
  const int gw = blockIdx.x * WPC + warp, nw = gridDim.x * WPC;
  auto issue = [&](int i, int s) {
    const uint8_t* g = src + ((size_t)i * nw + gw) * sbytes;
    uint8_t* d = st + (size_t)s * sbytes;
    if (mode == 0) {
      for (int c = lane; c < sbytes / 16; c += 32)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(sa(d + 16 * c)), "l"(g + 16 * c) : "memory");
      asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" :: "r"(sa(&bars[s])) : "memory");
    } else {
      const int bb = mode == 1 ? sbytes : sbytes - 256;
      if (lane == 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(sa(&bars[s])), "r"(bb) : "memory");
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                     :: "r"(sa(d)), "l"(g), "r"(bb), "r"(sa(&bars[s])) : "memory");
      }
      if (mode == 2) {
        if (lane < 16)
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(sa(d + bb + 16 * lane)), "l"(g + bb + 16 * lane) : "memory");
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" :: "r"(sa(&bars[s])) : "memory");
      }
    }
  };
  for (int s = 0; s < nst && s < items; ++s) issue(s, s);
  unsigned acc = 0;
  bool bad = false;
  for (int i = 0; i < items; ++i) {
    const int s = i % nst;
    if (!bad && !wait_b(&bars[s], (i / nst) & 1)) { bad = true; atomicOr(flag, 1u); }
    acc += reinterpret_cast<const unsigned*>(st + (size_t)s * sbytes)[lane];
    __syncwarp();
    if (!bad && i + nst < items) issue(i + nst, s);
  }
  if (bad) asm volatile("cp.async.wait_all;" ::: "memory");
  if (acc == 0x12345678u) sink[0] = acc;
}
int main() {
  const size_t total = (size_t)3 << 30;
  uint8_t* src; CK(cudaMalloc(&src, total)); CK(cudaMemset(src, 1, total));
  unsigned *flag, *sink; CK(cudaMalloc(&flag, 4)); CK(cudaMalloc(&sink, 4)); CK(cudaMemset(flag, 0, 4));
  CK(cudaFuncSetAttribute(stream, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024));
  cudaEvent_t e0, e1; cudaEventCreate(&e0); cudaEventCreate(&e1);
  struct Cfg { int wpc, mode, sb, nst; };
  const Cfg cfgs[] = {
    {1, 0, 4096, 8}, {1, 0, 8192, 8}, {1, 0, 16384, 8},
    {1, 1, 4096, 8}, {1, 1, 8192, 8}, {1, 1, 16384, 8}, {1, 1, 32768, 6},
    {2, 0, 4096, 8}, {2, 1, 4096, 8}, {2, 1, 8192, 8},
    {4, 0, 4096, 8}, {4, 1, 4096, 8}, {4, 1, 8192, 6},
  };
  for (const Cfg& c : cfgs) {
    const size_t smem = 2048 + (size_t)c.wpc * c.nst * c.sb;
    if (smem > 227 * 1024) { printf("skip\n"); continue; }
    const int items = (int)(total / ((size_t)148 * c.wpc * c.sb));
    stream<<<148, 32 * c.wpc, smem>>>(src, c.mode, c.sb, c.nst, items, flag, sink);
    CK(cudaDeviceSynchronize());
    cudaEventRecord(e0);
    stream<<<148, 32 * c.wpc, smem>>>(src, c.mode, c.sb, c.nst, items, flag, sink);
    cudaEventRecord(e1);
    CK(cudaEventSynchronize(e1));
    float ms; cudaEventElapsedTime(&ms, e0, e1);
    unsigned f; CK(cudaMemcpy(&f, flag, 4, cudaMemcpyDeviceToHost));
    const double bytes = (double)items * 148 * c.wpc * c.sb;
    printf("warps/CTA %d mode %d stage %6d B nst %d: %7.1f GB/s  (%.1f KB in flight/SM) flag=%u\n", c.wpc, c.mode, c.sb, c.nst,
           bytes / ms / 1e6, (double)c.wpc * c.nst * c.sb / 1024, f);
  }
  printf("done\n");
  return 0;
}
