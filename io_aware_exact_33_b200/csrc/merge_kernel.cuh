// merge_kernel.cuh - merge of partial attention results over disjoint key
// sets (split-KV decoding, sequence-parallel partials).
//
// For query row r with S parts, each computed over its own key set:
//     LSE_r = log sum_s exp(LSE_s,r),   O_r = sum_s exp(LSE_s,r - LSE_r) O_s,r
// (the identity the online softmax itself rests on); a row whose parts all
// have LSE = -inf gets O = 0 and LSE = -inf.  Memory-bound: each row reads
// S 16-bit O rows and S LSE values and writes one of each.
//
// Layout: o_parts (S, B, Nq, H, d) 16-bit, lse_parts (S, B, H, Nq) fp32;
// o (B, Nq, H, d), lse (B, H, Nq).  d / 8 lanes per row, one 16-byte
// vector of O per lane and part.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

namespace attn {

struct MergeParams {
  const uint16_t* o_parts;
  const float* lse_parts;
  uint16_t* o;
  float* lse;
  int splits, nq, nheads, headdim;
  long long rows;  // B * Nq * H
};

template <bool FP16>
__device__ __forceinline__ void unpack8(uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if constexpr (FP16) {
      f[2 * k] = __half2float(__ushort_as_half((unsigned short)(w[k] & 0xFFFFu)));
      f[2 * k + 1] = __half2float(__ushort_as_half((unsigned short)(w[k] >> 16)));
    } else {
      f[2 * k] = __uint_as_float(w[k] << 16);
      f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
}

template <bool FP16>
__device__ __forceinline__ uint32_t pack2_rn(float lo, float hi) {
  uint32_t r;
  if constexpr (FP16)
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  else
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <bool FP16>
__global__ void __launch_bounds__(256) attn_merge_kernel(const MergeParams p) {
  const int lpr = p.headdim / 8;  // lanes per row
  const int rpw = 32 / lpr;       // rows per warp step
  const int lane = threadIdx.x & 31, sub = lane % lpr;
  const long long warp_global = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const long long lrows = p.rows;  // LSE entries per part (B * H * Nq)
  for (long long r0 = warp_global * rpw; r0 < p.rows; r0 += nwarps * rpw) {
    const long long r = r0 + lane / lpr;
    if (r >= p.rows) continue;
    const long long h = r % p.nheads, i = (r / p.nheads) % p.nq, b = r / ((long long)p.nheads * p.nq);
    const long long lr = (b * p.nheads + h) * p.nq + i;
    float m = -INFINITY;
    for (int s = 0; s < p.splits; ++s) m = fmaxf(m, p.lse_parts[s * lrows + lr]);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float total = -INFINITY;
    if (m != -INFINITY) {
      float z = 0.f;
      for (int s = 0; s < p.splits; ++s) z += __expf(p.lse_parts[s * lrows + lr] - m);
      total = m + __logf(z);
      // parts in groups of four, their loads issued before any is used
      const uint16_t* base = p.o_parts + r * p.headdim + sub * 8;
      const long long part_stride = p.rows * p.headdim;
      for (int s0 = 0; s0 < p.splits; s0 += 4) {
        uint4 v[4];
        float w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int s = s0 + u;
          w[u] = s < p.splits ? __expf(p.lse_parts[s * lrows + lr] - total) : 0.f;
          v[u] = s < p.splits ? *reinterpret_cast<const uint4*>(base + s * part_stride)
                              : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float f[8];
          unpack8<FP16>(v[u], f);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = fmaf(w[u], f[e], acc[e]);
        }
      }
    }
    uint4 out;
    out.x = pack2_rn<FP16>(acc[0], acc[1]);
    out.y = pack2_rn<FP16>(acc[2], acc[3]);
    out.z = pack2_rn<FP16>(acc[4], acc[5]);
    out.w = pack2_rn<FP16>(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(p.o + r * p.headdim + sub * 8) = out;
    if (sub == 0) p.lse[lr] = total;
  }
}

}  // namespace attn
