// decode_kernel.cuh - attention of a few query rows against a long key /
// value sequence (decoding with a cache), split over the keys.
//
// With one to a few query tokens per sequence the work is reading K and V
// once: about R / 2 multiply-adds per byte for the R query rows that share a
// kv head, far below the tensor-core ridge, so this path runs on the CUDA
// cores and is bound by HBM.  One block per (key split, batch, kv head)
// takes all the query rows that read that kv head (the G query heads of the
// group times the Nq query tokens, R = G * Nq <= kDecodeRows), so every K and
// V row is read once for the whole group.  Each block writes its split's
// partial output (16-bit) and LSE; attn_merge combines the splits (the
// online-softmax rescale, as for split-KV calls of attn_fwd).
//
// Block: warp 8 is the producer, warps 0-7 compute.
//   * The producer streams the split's K and V in tiles of 64 keys through a
//     three-slot ring in shared memory (TMA, 128-byte swizzle, one mbarrier
//     per slot for "full" and one for "empty"), so the loads of the next
//     tiles are in flight while the current one is computed.
//   * Warp w takes keys 8w .. 8w + 7 of each tile, in two groups of four.
//     Scores: lane = 4 p + kk holds head-dim part p (D / 8 columns) of key
//     kk of the group; it reads its part of the K row from the swizzled tile
//     and of every query row from shared memory (queries pre-scaled by
//     softmax_scale * log2 e, fp32), and three shuffles sum the parts.
//   * Online softmax per query row over the warp's keys (running max and
//     sum), then O += P V with lane l owning head-dim columns
//     [l D/32, (l + 1) D/32) and P of each key taken by shuffle.
//   * At the end the eight warps' (max, sum, O) are combined through shared
//     memory (the ring, no longer needed) into the split's result.
// Products go through packed f32x2 FMAs.  Grid: the host picks the number of
// splits so that the blocks fill whole waves of the SMs.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

#include "merge_kernel.cuh"
#include "sm100.cuh"

namespace attn {

constexpr int kDecodeRows = 16;    // query rows per block at most: group size x query tokens
constexpr int kDecodeWarps = 8;    // compute warps
constexpr int kDecodeBN = 64;      // keys per tile
constexpr int kDecodeStages = 3;   // ring slots
constexpr int kDecodeThreads = (kDecodeWarps + 1) * 32;

struct DecodeParams {
  const uint16_t* q;  // (B, Nq, H, D)
  uint16_t* o_parts;  // (splits, B, Nq, H, D)
  float* lse_parts;   // (splits, B, H, Nq), natural log
  int batch, nheads, nheads_kv, seqlen_q, seqlen_k;
  int causal, window_left, window_right;
  float scale_log2;
  int splits;
  int key_lo;           // first key any query row can see
  int tiles_per_split;  // key tiles (kDecodeBN keys) of one split
  int tiles_total;      // key tiles from key_lo to the last visible key
};

template <int D>
struct DecodeCfg {
  static constexpr int NBOX = D / 64;                     // 64-column TMA boxes per row
  static constexpr int BOX_BYTES = kDecodeBN * 128;       // one box: 64 rows x 128 bytes
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;     // K or V tile
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;      // K then V
  static constexpr int COLS = D / 8;                      // head-dim columns of a score lane
  static constexpr int CPL = D / 32;                      // head-dim columns of an output lane
  static constexpr int OFF_Q = kDecodeStages * STAGE_BYTES;  // fp32 (kDecodeRows, D)
  static constexpr int OFF_BAR = OFF_Q + kDecodeRows * D * 4;
  static constexpr int B_FULL = 0, B_EMPTY = kDecodeStages, NBAR = 2 * kDecodeStages;
  static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 1024;
  // combine area (reuses the ring): per warp and row, O then (max, sum)
  static constexpr int COMB_O = 0;
  static constexpr int COMB_ML = kDecodeWarps * kDecodeRows * D * 4;
  static_assert(COMB_ML + kDecodeWarps * kDecodeRows * 8 <= OFF_Q, "combine area");
};

template <bool FP16>
__device__ __forceinline__ float half_to_float(uint16_t h) {
  if constexpr (FP16) return __half2float(__ushort_as_half(h));
  else return __uint_as_float((uint32_t)h << 16);
}

// Two 16-bit values of a 32-bit word as floats (low half first).
template <bool FP16>
__device__ __forceinline__ void unpack2(uint32_t w, float& lo, float& hi) {
  if constexpr (FP16) {
    lo = __half2float(__ushort_as_half((unsigned short)(w & 0xFFFFu)));
    hi = __half2float(__ushort_as_half((unsigned short)(w >> 16)));
  } else {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
  }
}

// RMAX: rows the registers are sized for (4, 8 or 16); R <= RMAX rows are live.
template <int D, bool FP16, int RMAX>
__global__ void __launch_bounds__(kDecodeThreads, (RMAX <= 8) ? 2 : 1)
    attn_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  using C = DecodeCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem0 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem0 - smem_addr(smem_raw));
  float* qs = reinterpret_cast<float*>(smem_gen + C::OFF_Q);
  auto bar = [&](int i) -> uint32_t { return smem0 + C::OFF_BAR + 8u * i; };

  const int split = blockIdx.y, bk = blockIdx.x;  // x: (batch, kv head)
  const int b = bk / p.nheads_kv, kvh = bk % p.nheads_kv;
  const int G = p.nheads / p.nheads_kv, Nq = p.seqlen_q, R = G * Nq;  // row r = g * Nq + i
  const uint32_t warp = warp_id(), lane = lane_id();

  // this split's key tiles
  const int t_begin = split * p.tiles_per_split;
  const int t_end = min(t_begin + p.tiles_per_split, p.tiles_total);
  const int ntiles = max(t_end - t_begin, 0);
  const int key0 = p.key_lo + t_begin * kDecodeBN;

  if (threadIdx.x == kDecodeWarps * 32) {
    for (int i = 0; i < C::NBAR; ++i) mbar_init(bar(i), i >= C::B_EMPTY ? kDecodeWarps : 1);
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  // queries, pre-scaled, as fp32 rows (rows R .. RMAX - 1 zero)
  for (int idx = threadIdx.x; idx < RMAX * D; idx += blockDim.x) {
    const int r = idx / D, c = idx % D;
    float x = 0.f;
    if (r < R) {
      const int g = r / Nq, i = r % Nq;
      x = half_to_float<FP16>(
              p.q[(((size_t)b * Nq + i) * p.nheads + (size_t)kvh * G + g) * D + c]) *
          p.scale_log2;
    }
    qs[idx] = x;
  }
  __syncthreads();

  if (warp == kDecodeWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && ntiles > 0) {
      bool go = true;
      for (int t = 0; go && t < ntiles; ++t) {
        const int st = t % kDecodeStages, n = t / kDecodeStages;
        if (n > 0 && !mbar_wait(bar(C::B_EMPTY + st), (n - 1) & 1)) { go = false; break; }
        const uint32_t base = smem0 + st * C::STAGE_BYTES;
        mbar_arrive_expect_tx(bar(C::B_FULL + st), C::STAGE_BYTES);
        for (int bx = 0; bx < C::NBOX; ++bx) {
          tma_load_4d(base + bx * C::BOX_BYTES, &tm_k, bar(C::B_FULL + st), bx * 64, kvh,
                      key0 + t * kDecodeBN, b);
          tma_load_4d(base + C::TILE_BYTES + bx * C::BOX_BYTES, &tm_v, bar(C::B_FULL + st),
                      bx * 64, kvh, key0 + t * kDecodeBN, b);
        }
      }
      // the block leaves only after its last loads have landed
      for (int t = max(ntiles - kDecodeStages, 0); go && t < ntiles; ++t)
        if (!mbar_wait(bar(C::B_FULL + t % kDecodeStages), (t / kDecodeStages) & 1)) break;
    }
  }

  // ------------------------------------------------------------ compute
  const long long off = (long long)p.seqlen_k - Nq;
  const long long kInf = 1ll << 40;
  const long long rb = p.causal ? 0 : (p.window_right >= 0 ? p.window_right : kInf);
  const long long lb = p.window_left >= 0 ? p.window_left : kInf;
  const int part = (int)(lane >> 2), kk = (int)(lane & 3);
  float m[RMAX], l[RMAX];
  uint64_t acc[RMAX][C::CPL / 2];  // column pairs of this lane's output columns
#pragma unroll
  for (int r = 0; r < RMAX; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int c = 0; c < C::CPL / 2; ++c) acc[r][c] = f2_pack(0.f, 0.f);
  }
  if (warp < kDecodeWarps) {
    for (int t = 0; t < ntiles; ++t) {
      const int st = t % kDecodeStages;
      // on expiry the status word reports the error; the warp stops reading
      if (!mbar_wait_warp(bar(C::B_FULL + st), (t / kDecodeStages) & 1)) break;
      const uint32_t kbase = smem0 + st * C::STAGE_BYTES;
      const uint32_t vbase = kbase + C::TILE_BYTES;
      const int jt = key0 + t * kDecodeBN;  // first key of the tile
      // scores of the warp's two groups of four keys: both groups' parts of
      // K first, so that each query load serves both
      float kf[2][C::COLS];  // this lane's D/8 columns of its two K rows
#pragma unroll
      for (int grp = 0; grp < 2; ++grp) {
        const int row = (int)warp * 8 + grp * 4 + kk;  // key within the tile
#pragma unroll
        for (int ch = 0; ch < C::COLS / 8; ++ch) {
          const int col = part * C::COLS + ch * 8;
          const int bx = col / 64, chunk = ((col % 64) / 8) ^ (row & 7);
          uint32_t w0, w1, w2, w3;
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3)
                       : "r"(kbase + bx * C::BOX_BYTES + row * 128 + chunk * 16));
          unpack2<FP16>(w0, kf[grp][ch * 8 + 0], kf[grp][ch * 8 + 1]);
          unpack2<FP16>(w1, kf[grp][ch * 8 + 2], kf[grp][ch * 8 + 3]);
          unpack2<FP16>(w2, kf[grp][ch * 8 + 4], kf[grp][ch * 8 + 5]);
          unpack2<FP16>(w3, kf[grp][ch * 8 + 6], kf[grp][ch * 8 + 7]);
        }
      }
      float s[2][RMAX];
#pragma unroll
      for (int r = 0; r < RMAX; ++r) {
        uint64_t s2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
        if (r < R) {
          const uint32_t qaddr = smem0 + C::OFF_Q + (r * D + part * C::COLS) * 4;
#pragma unroll
          for (int c4 = 0; c4 < C::COLS / 4; ++c4) {
            float q4[4];
            ld_shared_v4f(qaddr + c4 * 16, q4);
            const uint64_t qa = f2_pack(q4[0], q4[1]), qb = f2_pack(q4[2], q4[3]);
#pragma unroll
            for (int grp = 0; grp < 2; ++grp) {
              s2[grp] = f2_fma(qa, f2_pack(kf[grp][4 * c4], kf[grp][4 * c4 + 1]), s2[grp]);
              s2[grp] = f2_fma(qb, f2_pack(kf[grp][4 * c4 + 2], kf[grp][4 * c4 + 3]), s2[grp]);
            }
          }
        }
#pragma unroll
        for (int grp = 0; grp < 2; ++grp) {
          float e, o;
          f2_unpack(s2[grp], e, o);
          float x = e + o;
          x += __shfl_xor_sync(0xffffffffu, x, 4);
          x += __shfl_xor_sync(0xffffffffu, x, 8);
          x += __shfl_xor_sync(0xffffffffu, x, 16);
          // mask: key j of query i is visible iff i + off - lb <= j <= i + off + rb
          const long long j = (long long)jt + (int)warp * 8 + grp * 4 + kk;
          const long long i = r % Nq;
          const bool vis = r < R && j < p.seqlen_k && j <= i + off + rb && j >= i + off - lb;
          s[grp][r] = vis ? x : -INFINITY;
        }
      }
      // online softmax per row over the warp's eight keys, then O += P V
      float pr[2][RMAX];
#pragma unroll
      for (int r = 0; r < RMAX; ++r) {
        float mx = fmaxf(s[0][r], s[1][r]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_new = fmaxf(m[r], mx);
        float alpha = 1.f;
        pr[0][r] = pr[1][r] = 0.f;
        if (m_new != -INFINITY) {
          alpha = ex2(m[r] - m_new);  // 0 when m[r] = -inf
          pr[0][r] = ex2(s[0][r] - m_new);
          pr[1][r] = ex2(s[1][r] - m_new);
        }
        float sum = pr[0][r] + pr[1][r];
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        l[r] = l[r] * alpha + sum;
        m[r] = m_new;
        const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
        for (int c = 0; c < C::CPL / 2; ++c) acc[r][c] = f2_mul(acc[r][c], a2);
      }
#pragma unroll
      for (int key = 0; key < 8; ++key) {
        const int row = (int)warp * 8 + key;
        // this lane's CPL columns of the V row
        const int col = (int)lane * C::CPL;
        const int bx = col / 64, chunk = ((col % 64) / 8) ^ (row & 7);
        const uint32_t vaddr = vbase + bx * C::BOX_BYTES + row * 128 + chunk * 16 + (col % 8) * 2;
        float vf[C::CPL];
        if constexpr (C::CPL == 4) {
          uint32_t w0, w1;
          asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(w0), "=r"(w1) : "r"(vaddr));
          unpack2<FP16>(w0, vf[0], vf[1]);
          unpack2<FP16>(w1, vf[2], vf[3]);
        } else {
          uint32_t w0;
          asm volatile("ld.shared.b32 %0, [%1];" : "=r"(w0) : "r"(vaddr));
          unpack2<FP16>(w0, vf[0], vf[1]);
        }
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
          if (r < R) {
            const float pv = __shfl_sync(0xffffffffu, pr[key / 4][r], key % 4);
            const uint64_t p2 = f2_pack(pv, pv);
#pragma unroll
            for (int c = 0; c < C::CPL / 2; ++c)
              acc[r][c] = f2_fma(p2, f2_pack(vf[2 * c], vf[2 * c + 1]), acc[r][c]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_EMPTY + st));
    }
  }

  // ------------------------------------------------------------ combine
  __syncthreads();  // every warp is done with the ring: it becomes the combine area
  float* comb_o = reinterpret_cast<float*>(smem_gen + C::COMB_O);
  float* comb_ml = reinterpret_cast<float*>(smem_gen + C::COMB_ML);
  if (warp < kDecodeWarps) {
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
      if (r < R) {
#pragma unroll
        for (int c = 0; c < C::CPL / 2; ++c) {
          float lo, hi;
          f2_unpack(acc[r][c], lo, hi);
          comb_o[(warp * kDecodeRows + r) * D + lane * C::CPL + 2 * c] = lo;
          comb_o[(warp * kDecodeRows + r) * D + lane * C::CPL + 2 * c + 1] = hi;
        }
        if (lane == 0) {
          comb_ml[(warp * kDecodeRows + r) * 2] = m[r];
          comb_ml[(warp * kDecodeRows + r) * 2 + 1] = l[r];
        }
      }
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < R * D; idx += blockDim.x) {
    const int r = idx / D, c = idx % D, g = r / Nq, i = r % Nq, h = kvh * G + g;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) mx = fmaxf(mx, comb_ml[(w * kDecodeRows + r) * 2]);
    float sum = 0.f, o = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kDecodeWarps; ++w) {
        const float sc = ex2(comb_ml[(w * kDecodeRows + r) * 2] - mx);
        sum += comb_ml[(w * kDecodeRows + r) * 2 + 1] * sc;
        o += comb_o[(w * kDecodeRows + r) * D + c] * sc;
      }
    }
    const float ov = sum > 0.f ? o / sum : 0.f;
    const size_t part_i = ((size_t)split * p.batch + b);
    const size_t dst = ((part_i * Nq + i) * p.nheads + h) * D + c;
    p.o_parts[dst] = (uint16_t)(pack2_rn<FP16>(ov, 0.f) & 0xFFFFu);
    if (c == 0)
      p.lse_parts[(part_i * p.nheads + h) * Nq + i] =
          sum > 0.f ? (mx + __log2f(sum)) * 0.69314718055994530942f : -INFINITY;
  }
}

}  // namespace attn
