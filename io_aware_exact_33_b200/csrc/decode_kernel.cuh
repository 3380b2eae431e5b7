// decode_kernel.cuh - attention of a few query rows against a long key /
// value sequence (decoding with a cache), split over the keys.
//
// With one to a few query tokens per sequence the work is reading K and V
// once: about G / 2 multiply-adds per byte for a group of G query heads, far
// below the tensor-core ridge, so this path runs on the CUDA cores and is
// bound by HBM.  One block per (key split, batch, kv head) takes all the
// query rows that read that kv head (the G query heads of the group times
// the Nq query tokens, at most kDecodeRows), so every K and V row is read
// once for the whole group.  Each block writes its split's partial output
// (16-bit) and LSE; attn_merge combines the splits (the online-softmax
// rescale, as for split-KV calls of attn_fwd).
//
// Within a block each warp takes 32 keys at a time:
//   * scores: lane l owns key j0 + l, reads its K row (16-byte loads) and
//     forms the dot product with every query row (queries in shared memory,
//     pre-scaled by softmax_scale * log2 e, read as broadcasts);
//   * online softmax per row across the warp (shuffle max and sum), P of
//     the 32 keys staged in shared memory;
//   * O += P V: lane l owns head-dim columns [l * D/32, (l + 1) * D/32) and
//     reads each of the 32 V rows in one coalesced warp access.
// Products go through packed f32x2 FMAs (two head-dim columns each).
// The warps' running (max, sum, O) are combined in shared memory at the end.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

#include "merge_kernel.cuh"
#include "sm100.cuh"

namespace attn {

constexpr int kDecodeRows = 16;  // query rows per block: group size x query tokens
constexpr int kDecodeWarps = 8;

struct DecodeParams {
  const uint16_t* q;  // (B, Nq, H, D)
  const uint16_t* k;  // (B, Nk, Hkv, D)
  const uint16_t* v;
  uint16_t* o_parts;  // (splits, B, Nq, H, D)
  float* lse_parts;   // (splits, B, H, Nq), natural log
  int batch, nheads, nheads_kv, seqlen_q, seqlen_k;
  int causal, window_left, window_right;
  float scale_log2;
  int splits, chunk;  // keys per split (a multiple of 32)
};

template <int D>
struct DecodeSmem {
  static constexpr int Q = kDecodeRows * D;                    // scaled queries
  static constexpr int P = kDecodeWarps * kDecodeRows * 32;    // P of each warp's 32 keys
  static constexpr int O = kDecodeWarps * kDecodeRows * D;     // each warp's partial O
  static constexpr int ML = kDecodeWarps * kDecodeRows * 2;    // each warp's max and sum
  static constexpr int BYTES = (Q + P + O + ML) * 4;
};

template <bool FP16>
__device__ __forceinline__ float half_to_float(uint16_t h) {
  if constexpr (FP16) return __half2float(__ushort_as_half(h));
  else return __uint_as_float((uint32_t)h << 16);
}

template <int D, bool FP16>
__global__ void __launch_bounds__(kDecodeWarps * 32) attn_decode_kernel(const DecodeParams p) {
  constexpr int CPL = D / 32;  // head-dim columns per lane in the P V product
  using S = DecodeSmem<D>;
  extern __shared__ float smem_f[];
  float* qs = smem_f;
  float* ps = qs + S::Q;
  float* os = ps + S::P;
  float* mls = os + S::O;

  const int split = blockIdx.y, bk = blockIdx.x;  // x: (batch, kv head), up to 2^31 - 1
  const int b = bk / p.nheads_kv, kvh = bk % p.nheads_kv;
  const int G = p.nheads / p.nheads_kv, Nq = p.seqlen_q, R = G * Nq;  // row r = g * Nq + i
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int idx = threadIdx.x; idx < R * D; idx += blockDim.x) {
    const int r = idx / D, c = idx % D, g = r / Nq, i = r % Nq;
    const size_t src = (((size_t)b * Nq + i) * p.nheads + (size_t)kvh * G + g) * D + c;
    qs[idx] = half_to_float<FP16>(p.q[src]) * p.scale_log2;
  }
  __syncthreads();

  const int k_begin = split * p.chunk;
  const int k_end = min(k_begin + p.chunk, p.seqlen_k);
  const long long off = (long long)p.seqlen_k - Nq;
  const long long kInf = 1ll << 40;
  const long long rb = p.causal ? 0 : (p.window_right >= 0 ? p.window_right : kInf);
  const long long lb = p.window_left >= 0 ? p.window_left : kInf;
  const size_t row_stride = (size_t)p.nheads_kv * D;  // elements between consecutive keys
  const uint16_t* kbase = p.k + ((size_t)b * p.seqlen_k * p.nheads_kv + kvh) * D;
  const uint16_t* vbase = p.v + ((size_t)b * p.seqlen_k * p.nheads_kv + kvh) * D;

  float m[kDecodeRows], l[kDecodeRows];
  uint64_t acc[kDecodeRows][CPL / 2];  // column pairs of this lane's O rows
#pragma unroll
  for (int r = 0; r < kDecodeRows; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int c = 0; c < CPL / 2; ++c) acc[r][c] = f2_pack(0.f, 0.f);
  }

  for (int j0 = k_begin + warp * 32; j0 < k_end; j0 += kDecodeWarps * 32) {
    const int j = j0 + lane;
    float s[kDecodeRows];
    {
      uint64_t s2[kDecodeRows];  // (even, odd) column partial sums
#pragma unroll
      for (int r = 0; r < kDecodeRows; ++r) s2[r] = f2_pack(0.f, 0.f);
      if (j < k_end) {
        const uint4* krow = reinterpret_cast<const uint4*>(kbase + (size_t)j * row_stride);
#pragma unroll 4
        for (int c8 = 0; c8 < D / 8; ++c8) {
          float kf[8];
          unpack8<FP16>(__ldg(krow + c8), kf);
          const uint64_t k01 = f2_pack(kf[0], kf[1]), k23 = f2_pack(kf[2], kf[3]);
          const uint64_t k45 = f2_pack(kf[4], kf[5]), k67 = f2_pack(kf[6], kf[7]);
#pragma unroll
          for (int r = 0; r < kDecodeRows; ++r) {
            if (r < R) {
              const float4 qa = *reinterpret_cast<const float4*>(qs + r * D + c8 * 8);
              const float4 qb = *reinterpret_cast<const float4*>(qs + r * D + c8 * 8 + 4);
              s2[r] = f2_fma(f2_pack(qa.x, qa.y), k01, s2[r]);
              s2[r] = f2_fma(f2_pack(qa.z, qa.w), k23, s2[r]);
              s2[r] = f2_fma(f2_pack(qb.x, qb.y), k45, s2[r]);
              s2[r] = f2_fma(f2_pack(qb.z, qb.w), k67, s2[r]);
            }
          }
        }
      }
#pragma unroll
      for (int r = 0; r < kDecodeRows; ++r) {
        float e, o;
        f2_unpack(s2[r], e, o);
        s[r] = e + o;
      }
    }
    // masks: key j of query i is visible iff i + off - lb <= j <= i + off + rb
#pragma unroll
    for (int r = 0; r < kDecodeRows; ++r) {
      if (r < R) {
        const long long i = r % Nq;
        const bool vis = j < k_end && (long long)j <= i + off + rb && (long long)j >= i + off - lb;
        if (!vis) s[r] = -INFINITY;
      }
    }
    // online softmax of the warp's 32 keys, row by row
    float* pw = ps + warp * kDecodeRows * 32;
#pragma unroll
    for (int r = 0; r < kDecodeRows; ++r) {
      if (r < R) {
        float mx = s[r];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float m_new = fmaxf(m[r], mx);
        float pr = 0.f, alpha = 1.f;
        if (m_new != -INFINITY) {
          pr = exp2f(s[r] - m_new);
          alpha = exp2f(m[r] - m_new);  // 0 when m[r] = -inf
        }
        float sum = pr;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        l[r] = l[r] * alpha + sum;
        m[r] = m_new;
        const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
        for (int c = 0; c < CPL / 2; ++c) acc[r][c] = f2_mul(acc[r][c], a2);
        pw[r * 32 + lane] = pr;
      }
    }
    __syncwarp();
    const int nkeys = min(32, k_end - j0);
    for (int jj = 0; jj < nkeys; ++jj) {
      const uint16_t* vrow = vbase + (size_t)(j0 + jj) * row_stride + lane * CPL;
      float vf[CPL];
      if constexpr (CPL == 4) {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(vrow));
        vf[0] = half_to_float<FP16>((uint16_t)(w.x & 0xFFFFu));
        vf[1] = half_to_float<FP16>((uint16_t)(w.x >> 16));
        vf[2] = half_to_float<FP16>((uint16_t)(w.y & 0xFFFFu));
        vf[3] = half_to_float<FP16>((uint16_t)(w.y >> 16));
      } else {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(vrow));
        vf[0] = half_to_float<FP16>((uint16_t)(w & 0xFFFFu));
        vf[1] = half_to_float<FP16>((uint16_t)(w >> 16));
      }
#pragma unroll
      for (int r = 0; r < kDecodeRows; ++r) {
        if (r < R) {
          const float pr = pw[r * 32 + jj];
          const uint64_t p2 = f2_pack(pr, pr);
#pragma unroll
          for (int c = 0; c < CPL / 2; ++c)
            acc[r][c] = f2_fma(p2, f2_pack(vf[2 * c], vf[2 * c + 1]), acc[r][c]);
        }
      }
    }
    __syncwarp();
  }

  // combine the warps' running states
#pragma unroll
  for (int r = 0; r < kDecodeRows; ++r) {
    if (r < R) {
#pragma unroll
      for (int c = 0; c < CPL / 2; ++c) {
        float lo, hi;
        f2_unpack(acc[r][c], lo, hi);
        os[(warp * kDecodeRows + r) * D + lane * CPL + 2 * c] = lo;
        os[(warp * kDecodeRows + r) * D + lane * CPL + 2 * c + 1] = hi;
      }
      if (lane == 0) {
        mls[(warp * kDecodeRows + r) * 2] = m[r];
        mls[(warp * kDecodeRows + r) * 2 + 1] = l[r];
      }
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < R * D; idx += blockDim.x) {
    const int r = idx / D, c = idx % D, g = r / Nq, i = r % Nq, h = kvh * G + g;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) mx = fmaxf(mx, mls[(w * kDecodeRows + r) * 2]);
    float sum = 0.f, o = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kDecodeWarps; ++w) {
        const float sc = exp2f(mls[(w * kDecodeRows + r) * 2] - mx);
        sum += mls[(w * kDecodeRows + r) * 2 + 1] * sc;
        o += os[(w * kDecodeRows + r) * D + c] * sc;
      }
    }
    const float ov = sum > 0.f ? o / sum : 0.f;
    const size_t part = ((size_t)split * p.batch + b);
    const size_t dst = ((part * Nq + i) * p.nheads + h) * D + c;
    if constexpr (FP16) p.o_parts[dst] = __half_as_ushort(__float2half_rn(ov));
    else p.o_parts[dst] = (uint16_t)(pack2_rn<false>(ov, 0.f) & 0xFFFFu);
    if (c == 0)
      p.lse_parts[(part * p.nheads + h) * Nq + i] =
          sum > 0.f ? (mx + __log2f(sum)) * 0.69314718055994530942f : -INFINITY;
  }
}

}  // namespace attn
