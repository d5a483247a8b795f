// HBM streaming-read probe (a standalone measurement program, not part of the
// library): which way of reading global memory saturates HBM on this GPU?
//  A: 1-D bulk copies (cp.async.bulk, TMA) of `copy` bytes into a ring of
//     `ring` shared-memory slots, issued by one producer thread per CTA, with
//     full/empty mbarriers (bounded waits);
//  B: 128-bit loads (ld.global.cs), U independent loads in flight per thread.
// Reads 4 GiB per launch, best of 3, CUDA events.
// Build: nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 \
//          -o hbm_stream_probe hbm_stream_probe.cu
#include <cuda_runtime.h>
#include <cstdio>
#include <cstdint>
#include <vector>

__device__ __forceinline__ uint32_t su(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__global__ void __launch_bounds__(288, 1) tma_ring(const unsigned char* buf, size_t bytes_per_cta,
                                                   int copy_bytes, int ring, unsigned* out, unsigned* err) {
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t* full = (uint64_t*)(smem + (size_t)ring * copy_bytes);
  uint64_t* empty = full + ring;
  const unsigned char* base = buf + (size_t)blockIdx.x * bytes_per_cta;
  const int n = (int)(bytes_per_cta / copy_bytes);
  if (threadIdx.x == 0) {
    for (int s = 0; s < ring; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su(&full[s])), "r"(1));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su(&empty[s])), "r"(8));
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  unsigned acc = 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 8) {
    if (lane == 0) {
      for (int i = 0; i < n; ++i) {
        int slot = i % ring, use = i / ring;
        if (use > 0) {
          uint32_t ok = 0; long long spins = 0;
          while (!ok && spins < (1ll << 26)) {
            asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0,1,0,p; }"
                         : "=r"(ok) : "r"(su(&empty[slot])), "r"((use - 1) & 1) : "memory");
            ++spins;
          }
          if (!ok) { atomicOr(err, 1u); break; }
        }
        asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }"
                     ::"r"(su(&full[slot])), "r"(copy_bytes) : "memory");
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                     ::"r"(su(smem + (size_t)slot * copy_bytes)), "l"(base + (size_t)i * copy_bytes),
                     "r"(copy_bytes), "r"(su(&full[slot])) : "memory");
      }
    }
  } else {
    for (int i = 0; i < n; ++i) {
      int slot = i % ring, use = i / ring;
      uint32_t ok = 0; long long spins = 0;
      while (!ok && spins < (1ll << 26)) {
        asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0,1,0,p; }"
                     : "=r"(ok) : "r"(su(&full[slot])), "r"(use & 1) : "memory");
        ++spins;
      }
      if (!ok) { atomicOr(err, 2u); break; }
      const uint4* s = (const uint4*)(smem + (size_t)slot * copy_bytes);
      for (int j = threadIdx.x; j < copy_bytes / 16; j += 256) { uint4 v = s[j]; acc ^= v.x ^ v.w; }
      __syncwarp();
      if (lane == 0) asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(su(&empty[slot])) : "memory");
    }
  }
  if (acc == 0x12345678u) out[0] = acc;
}

template <int U>
__global__ void ldg_stream(const uint4* buf, size_t n16, unsigned* out) {
  unsigned acc = 0;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + (U - 1) * stride < n16; i += U * stride) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) v[u] = __ldcs(buf + i + u * stride);
#pragma unroll
    for (int u = 0; u < U; ++u) acc ^= v[u].x ^ v[u].w;
  }
  for (; i < n16; i += stride) { uint4 v = buf[i]; acc ^= v.x; }
  if (acc == 0x12345678u) out[0] = acc;
}

int main() {
  const size_t bytes = 4ull << 30;  // 4 GiB read per launch
  unsigned char* buf; unsigned *out, *err;
  if (cudaMalloc(&buf, bytes) != cudaSuccess) { printf("alloc failed\n"); return 1; }
  cudaMemset(buf, 1, bytes);
  cudaMalloc(&out, 64); cudaMalloc(&err, 64); cudaMemset(err, 0, 64);
  int sms = 0; cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  cudaEvent_t e0, e1; cudaEventCreate(&e0); cudaEventCreate(&e1);
  cudaFuncSetAttribute(tma_ring, cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
  int copies[] = {2048, 4096, 8192, 16384, 32768};
  int rings[] = {4, 8, 16, 32, 64};
  for (int ctas_per_sm : {1, 2}) {
    for (int cb : copies) for (int r : rings) {
      size_t smem = (size_t)cb * r + 2 * 8 * r;
      if (smem > (ctas_per_sm == 1 ? 200 * 1024 : 100 * 1024)) continue;
      int grid = sms * ctas_per_sm;
      size_t per = (bytes / grid) / cb * cb;
      float best = 1e9;
      for (int rep = 0; rep < 3; ++rep) {
        cudaEventRecord(e0);
        tma_ring<<<grid, 288, smem>>>(buf, per, cb, r, out, err);
        cudaEventRecord(e1); cudaEventSynchronize(e1);
        float ms; cudaEventElapsedTime(&ms, e0, e1); if (ms < best) best = ms;
      }
      unsigned herr = 0; cudaMemcpy(&herr, err, 4, cudaMemcpyDeviceToHost);
      printf("TMA ctas/sm=%d copy=%6d ring=%2d inflight/SM=%7d : %.1f GB/s err=%u %s\n", ctas_per_sm, cb, r,
             cb * r * ctas_per_sm, per * grid / (best * 1e-3) / 1e9, herr, cudaGetErrorString(cudaGetLastError()));
    }
  }
  for (int threads : {256, 512, 1024}) for (int bps : {1, 2, 4}) {
    if (threads * bps > 2048) continue;
    int grid = sms * bps;
    float best = 1e9;
    for (int u : {4, 8, 16}) {
      best = 1e9;
      for (int rep = 0; rep < 3; ++rep) {
        cudaEventRecord(e0);
        if (u == 4) ldg_stream<4><<<grid, threads>>>((const uint4*)buf, bytes / 16, out);
        if (u == 8) ldg_stream<8><<<grid, threads>>>((const uint4*)buf, bytes / 16, out);
        if (u == 16) ldg_stream<16><<<grid, threads>>>((const uint4*)buf, bytes / 16, out);
        cudaEventRecord(e1); cudaEventSynchronize(e1);
        float ms; cudaEventElapsedTime(&ms, e0, e1); if (ms < best) best = ms;
      }
      printf("LDG threads=%4d blocks/sm=%d U=%2d : %.1f GB/s %s\n", threads, bps, u, bytes / (best * 1e-3) / 1e9,
             cudaGetErrorString(cudaGetLastError()));
    }
  }
  return 0;
}
