// probe_mma.cu - tcgen05.mma throughput by shape and operand source.
//
// Measurement tool, not part of libattn.so: one CTA per SM, one thread issues
// a long run of MMAs of a fixed shape (descriptors built once, stepped with
// adds), and clock64 gives cycles per instruction.  Used to choose the
// attention kernels' tile shapes: compare with M*N*16/4096 cycles, the
// dense bf16 rate of 4096 multiply-adds per clock per SM.
//
// Operands live in a zeroed 64 KB shared-memory area: A in the first 32 KB,
// B in the second; four K-steps stay inside one 128-byte-wide box (A at most
// 24 KB, B at most 32 KB), so every descriptor read is in bounds.
#include <cuda_runtime.h>
#include <stdint.h>

#include "sm100.cuh"

using namespace attn;

template <int M, int N, bool A_TMEM, bool A_MN, bool B_MN, int NACC>
__global__ void __launch_bounds__(128, 1) probe_mma_kernel(int iters, unsigned long long* out) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t s0 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  const uint32_t bar = s0 + 65536 + 1024;
  const uint32_t tptr = bar + 16;
  for (int i = threadIdx.x; i < 65536 / 16; i += blockDim.x) st_shared_v4(s0 + i * 16, 0, 0, 0, 0);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  if (threadIdx.x < 32) {
    tmem_alloc(tptr, 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  uint32_t tmem;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem) : "r"(tptr));
  if (threadIdx.x == 0) {
    constexpr uint32_t idesc = idesc_f16(M, N, false, A_MN, B_MN);
    uint64_t ad[4], bd[4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      ad[kk] = sdesc_sw128(s0 + (A_MN ? kk * 2048 : kk * 32), A_MN ? 16384 : 16, 1024);
      bd[kk] = sdesc_sw128(s0 + 32768 + (B_MN ? kk * 2048 : kk * 32), B_MN ? 8192 : 16, 1024);
    }
    const unsigned long long t0 = clock64();
    for (int it = 0; it < iters; it += 4 * NACC) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
        for (int a = 0; a < NACC; ++a) {
          // accumulators of 128 columns; A from tensor memory uses columns 0-31
          const uint32_t dcol = NACC == 1 ? 256 : (A_TMEM ? 128 + 128 * a : 128 * a);
          if (A_TMEM)
            mma_ts(tmem + dcol, tmem + kk * 8, bd[kk], idesc, 1u);
          else
            mma_ss(tmem + dcol, ad[kk], bd[kk], idesc, 1u);
        }
      }
    }
    mma_commit(bar);
    mbar_wait(bar, 0);
    out[blockIdx.x] = clock64() - t0;
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int M, int N, bool AT, bool AM, bool BM, int NACC>
int launch_probe(int iters, unsigned long long* out) {
  const int smem = 65536 + 1024 + 64 + 1024;
  auto k = probe_mma_kernel<M, N, AT, AM, BM, NACC>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return -2;
  k<<<148, 128, smem>>>(iters, out);
  return (int)cudaGetLastError();
}

// Case table shared with bench.py --probe-mma (same order).
extern "C" __attribute__((visibility("default"))) int probe_mma_case(int id, int iters,
                                                                     unsigned long long* out) {
  switch (id) {
    case 0: return launch_probe<128, 128, false, false, false, 1>(iters, out);
    case 1: return launch_probe<128, 128, false, false, false, 2>(iters, out);
    case 2: return launch_probe<128, 64, false, false, false, 1>(iters, out);
    case 3: return launch_probe<128, 64, false, false, false, 2>(iters, out);
    case 4: return launch_probe<128, 256, false, false, false, 1>(iters, out);
    case 5: return launch_probe<128, 64, false, true, true, 1>(iters, out);
    case 6: return launch_probe<128, 128, false, false, true, 1>(iters, out);
    case 7: return launch_probe<128, 128, true, false, true, 1>(iters, out);
    case 8: return launch_probe<128, 64, true, false, false, 1>(iters, out);
    case 9: return launch_probe<128, 256, true, false, true, 1>(iters, out);
    default: return -1;
  }
}
