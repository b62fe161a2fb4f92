// Probe: per-SM throughput of mma.sync bf16 m16n8k16, int8 m16n8k32, LOP3, and their overlap.
// 8 warps per CTA, 148 CTAs, register-only loops; results into a small buffer.
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
#define CK(x) do { cudaError_t e = (x); if (e != cudaSuccess) { printf("CUDA %s: %s\n", #x, cudaGetErrorString(e)); return 1; } } while (0)

template <int MODE, int NLOP>
__global__ void __launch_bounds__(256, 1) kern(uint32_t seed, int iters, float* out) {
  uint32_t a[8][4], b0 = seed ^ threadIdx.x, b1 = seed * 3u + threadIdx.x;
  float d[8][4];
  int di[8][4];
  for (int i = 0; i < 8; ++i) for (int j = 0; j < 4; ++j) { a[i][j] = seed + i * 7 + j; d[i][j] = 0.f; di[i][j] = 0; }
  uint32_t w = seed ^ (threadIdx.x * 77u);
  uint32_t x = 0;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (NLOP > 0) {
#pragma unroll
        for (int l = 0; l < NLOP; ++l) {
          uint32_t r;
          asm volatile("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w + l), "r"(0x000F000Fu << (l & 3)), "r"(0x43004300u));
          a[i][l & 3] ^= r;
        }
      }
      if (MODE == 1)
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                     : "+f"(d[i][0]), "+f"(d[i][1]), "+f"(d[i][2]), "+f"(d[i][3])
                     : "r"(a[i][0]), "r"(a[i][1]), "r"(a[i][2]), "r"(a[i][3]), "r"(b0), "r"(b1));
      if (MODE == 2)
        asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                     : "+r"(di[i][0]), "+r"(di[i][1]), "+r"(di[i][2]), "+r"(di[i][3])
                     : "r"(a[i][0]), "r"(a[i][1]), "r"(a[i][2]), "r"(a[i][3]), "r"(b0), "r"(b1));
      if (MODE == 3)
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                     : "+f"(d[i][0]), "+f"(d[i][1]), "+f"(d[i][2]), "+f"(d[i][3])
                     : "r"(a[i][0]), "r"(a[i][1]), "r"(a[i][2]), "r"(a[i][3]), "r"(b0), "r"(b1));
    }
    w = w * 1664525u + 1013904223u;
  }
  float s = 0.f;
  for (int i = 0; i < 8; ++i) for (int j = 0; j < 4; ++j) { s += d[i][j] + (float)di[i][j]; x ^= a[i][j]; }
  if (s == 1.2345f && x == 7u) out[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

template <int MODE, int NLOP>
int run(const char* name, float* out) {
  const int iters = 4096;
  cudaEvent_t e0, e1; cudaEventCreate(&e0); cudaEventCreate(&e1);
  kern<MODE, NLOP><<<148, 256>>>(1u, iters, out);
  CK(cudaDeviceSynchronize());
  cudaEventRecord(e0);
  kern<MODE, NLOP><<<148, 256>>>(2u, iters, out);
  cudaEventRecord(e1);
  CK(cudaEventSynchronize(e1));
  float ms; cudaEventElapsedTime(&ms, e0, e1);
  int clk; cudaDeviceGetAttribute(&clk, cudaDevAttrClockRate, 0);
  const double cycles = ms * 1e-3 * clk * 1e3;
  const double per_part = (double)iters * 8 * 2;  // 8 ops per iteration per warp, 2 warps per partition
  printf("%-28s %.3f ms, %.2f cycles per (MMA slot) per partition (@%d MHz max)\n", name, ms, cycles / per_part, clk / 1000);
  return 0;
}

int main() {
  float* out; CK(cudaMalloc(&out, 148 * 256 * 4));
  run<1, 0>("bf16 mma only", out);
  run<2, 0>("int8 k32 mma only", out);
  run<3, 0>("f16 mma only", out);
  run<0, 4>("4 lop3 only", out);
  run<0, 8>("8 lop3 only", out);
  run<1, 4>("bf16 mma + 4 lop3", out);
  run<1, 8>("bf16 mma + 8 lop3", out);
  run<2, 4>("int8 mma + 4 lop3", out);
  run<2, 8>("int8 mma + 8 lop3", out);
  printf("done\n");
  return 0;
}
