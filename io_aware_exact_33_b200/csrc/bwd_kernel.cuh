// bwd_kernel.cuh - exact attention backward pass for sm_100a.
//
// The backward pass recomputes the score tiles from Q, K and the saved
// log-sum-exp instead of storing them ("FlashAttention ... transformer
// optimization", item 2).  With P = exp(S*scale - LSE), dP = dO V^T and
// Dvec_i = rowsum(dO_i o O_i) (= sum_j P_ij dP_ij):
//     dV = P^T dO,   dS = P o (dP - Dvec),   dK = scale dS^T Q,   dQ = scale dS K.
//
// Three kernels:
//   bwd_preprocess  Dvec = rowsum(dO o O) (fp32), LSE in base 2 (+inf for a
//                   query with no visible key or a padding row) and a zeroed
//                   fp32 dQ accumulator, all in the caller's workspace.
//   attn_bwd_kernel one CTA per (batch, kv head, 128-key tile): K_j and V_j
//                   stay in shared memory and dK_j, dV_j accumulate in tensor
//                   memory while the CTA walks every query tile of every query
//                   head of the GQA group that sees the key tile.
//   bwd_convert     dQ = scale * accumulator, rounded to the input dtype.
//
// Main kernel roles (320 threads):
//   warp 8      TMA producer: K_j, V_j once; Q_i, dO_i, LSE2_i, Dvec_i per
//               query tile through a two-slot ring.
//   warp 9      TMEM allocation; lane 0 issues the five MMAs per tile:
//               S^T = K Q^T, dP^T = V dO^T, dV += P^T dO, dK += dS^T Q, and
//               dQ^T = K^T dS^T (d = 128) or dQ = dS K (d = 64).
//   warps 0-3   one thread per key row (TMEM lane): P^T = exp2(S^T*scale*log2e
//               - LSE2), dS^T = P^T o (dP^T - Dvec); P^T and dS^T go back to
//               TMEM as 16-bit operands, dS also to shared memory (the dQ MMA
//               needs it with the other operand order); finally dK, dV out.
//   warps 4-7   read the dQ tile out of TMEM and add it into the fp32
//               accumulator with global atomics (other key tiles add too).
#pragma once

#include <cuda_fp16.h>

#include "sm100.cuh"

namespace attn {

struct BwdWorkspace {
  size_t dvec_off, lse2_off, dq_off, total;
  long long nq_pad;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace: Dvec and LSE2 as (batch*nheads, nq_pad) fp32 with nq_pad a
// multiple of 128 (TMA-aligned rows), then the fp32 dQ accumulator
// (batch, seqlen_q, nheads, headdim).
__host__ __device__ inline BwdWorkspace bwd_workspace_layout(int batch, int nheads, int seqlen_q,
                                                            int headdim) {
  BwdWorkspace w;
  w.nq_pad = ((long long)seqlen_q + 127) / 128 * 128;
  const size_t rows = (size_t)batch * nheads * (size_t)w.nq_pad * 4;
  w.dvec_off = 0;
  w.lse2_off = align_up(rows, 256);
  w.dq_off = w.lse2_off + align_up(rows, 256);
  w.total = w.dq_off + align_up((size_t)batch * seqlen_q * nheads * headdim * 4, 256);
  return w;
}

struct BwdParams {
  const float* lse;
  float* dvec;
  float* lse2;
  float* dq_acc;
  int batch, nheads, nheads_kv, seqlen_q, seqlen_k, headdim;
  int causal, window_left, window_right;
  float scale_log2;
  float softmax_scale;
  long long nq_pad;
};

// ------------------------------------------------------------ preprocess
// One warp per (b, h, i) row of the padded range: Dvec_i = sum_c dO_ic O_ic,
// LSE2_i = LSE_i * log2(e).  Blocks past the rows zero the dQ accumulator.
template <bool FP16>
__global__ void __launch_bounds__(256) bwd_preprocess(const uint16_t* __restrict__ o,
                                                      const uint16_t* __restrict__ dout,
                                                      BwdParams p, long long n_rows,
                                                      long long n_zero4) {
  const long long warp_global = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long row = warp_global; row < n_rows; row += nwarps) {
    const long long i = row % p.nq_pad;
    const long long bh = row / p.nq_pad;
    const int h = (int)(bh % p.nheads), b = (int)(bh / p.nheads);
    float dv = 0.f, l2 = INFINITY;
    if (i < p.seqlen_q) {
      const size_t base = (((size_t)b * p.seqlen_q + i) * p.nheads + h) * p.headdim;
      float acc = 0.f;
      for (int c = lane * 2; c < p.headdim; c += 64) {
        const uint32_t ov = *reinterpret_cast<const uint32_t*>(o + base + c);
        const uint32_t dov = *reinterpret_cast<const uint32_t*>(dout + base + c);
        float o0, o1, d0, d1;
        if constexpr (FP16) {
          o0 = __half2float(__ushort_as_half((unsigned short)(ov & 0xFFFFu)));
          o1 = __half2float(__ushort_as_half((unsigned short)(ov >> 16)));
          d0 = __half2float(__ushort_as_half((unsigned short)(dov & 0xFFFFu)));
          d1 = __half2float(__ushort_as_half((unsigned short)(dov >> 16)));
        } else {
          o0 = __uint_as_float(ov << 16);
          o1 = __uint_as_float(ov & 0xFFFF0000u);
          d0 = __uint_as_float(dov << 16);
          d1 = __uint_as_float(dov & 0xFFFF0000u);
        }
        acc = fmaf(o0, d0, acc);
        acc = fmaf(o1, d1, acc);
      }
#pragma unroll
      for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
      dv = acc;
      const float l = p.lse[((size_t)b * p.nheads + h) * p.seqlen_q + i];
      l2 = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
    }
    if (lane == 0) {
      p.dvec[row] = dv;
      p.lse2[row] = l2;
    }
  }
  float4* z = reinterpret_cast<float4*>(p.dq_acc);
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  for (long long k = tid; k < n_zero4; k += nthreads) z[k] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ------------------------------------------------------------ convert
template <bool FP16>
__global__ void __launch_bounds__(256) bwd_convert(const float* __restrict__ acc,
                                                   uint16_t* __restrict__ dq, long long n4,
                                                   float scale) {
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  for (long long k = tid; k < n4; k += nthreads) {
    const float4 a = reinterpret_cast<const float4*>(acc)[k];
    uint2 w;
    w.x = pack2<FP16>(a.x * scale, a.y * scale);
    w.y = pack2<FP16>(a.z * scale, a.w * scale);
    reinterpret_cast<uint2*>(dq)[k] = w;
  }
}

// ------------------------------------------------------------ main kernel
template <int D_, bool FP16_>
struct BwdCfg {
  static constexpr int D = D_;
  static constexpr bool FP16 = FP16_;
  static constexpr int BN = 128;                 // key rows per CTA (TMEM lanes)
  static constexpr int BM = (D == 128) ? 64 : 128;  // query rows per step
  static constexpr bool DQT = (D == 128);        // dQ^T = K^T dS^T, else dQ = dS K
  static constexpr int NBOX = D / 64;
  static constexpr int NQB = BM / 64;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int DS_BYTES = BN * BM * 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_BYTES;
  static constexpr int OFF_Q = OFF_V + KV_BYTES;      // 2 slots
  static constexpr int OFF_DO = OFF_Q + 2 * Q_BYTES;  // 2 slots
  static constexpr int OFF_DS = OFF_DO + 2 * Q_BYTES;
  static constexpr int OFF_LSE = OFF_DS + DS_BYTES;   // 2 slots x BM fp32
  static constexpr int OFF_DVEC = OFF_LSE + 2 * BM * 4;
  static constexpr int OFF_BAR = OFF_DVEC + 2 * BM * 4;
  static constexpr int B_KV = 0;
  static constexpr int B_QFULL = 1;     // 2
  static constexpr int B_DOFULL = 3;    // 2
  static constexpr int B_EMPTY = 5;     // 2
  static constexpr int B_SFULL = 7;
  static constexpr int B_DPFULL = 8;
  static constexpr int B_PREADY = 9;    // 128 arrivals
  static constexpr int B_DSREADY = 10;  // 128 arrivals
  static constexpr int B_DSFREE = 11;
  static constexpr int B_DQFULL = 12;
  static constexpr int B_DQFREE = 13;   // 128 arrivals
  static constexpr int B_DONE = 14;
  static constexpr int NBAR = 15;
  static constexpr int OFF_TMEMPTR = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_TMEMPTR + 16 + 1024;
  static constexpr int TM_DV = 0, TM_DK = D, TM_S = 2 * D, TM_DP = 2 * D + BM, TM_DQ = 2 * D + 2 * BM;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 320;
  static_assert(TM_DQ + (DQT ? BM : D) <= TMEM_COLS, "tensor memory");
  static_assert(2 * Q_BYTES >= BN * D * 2, "epilogue staging");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_lse2, const __grid_constant__ CUtensorMap tm_dvec,
                    const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                    const BwdParams p) {
  constexpr int D = C::D, BN = C::BN, BM = C::BM;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem0 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem0 - smem_addr(smem_raw));
  auto bar = [&](int i) -> uint32_t { return smem0 + C::OFF_BAR + 8u * i; };
  volatile uint32_t* tmem_ptr_slot = reinterpret_cast<volatile uint32_t*>(smem_gen + C::OFF_TMEMPTR);
  const float* lse_s = reinterpret_cast<const float*>(smem_gen + C::OFF_LSE);
  const float* dvec_s = reinterpret_cast<const float*>(smem_gen + C::OFF_DVEC);

  const uint32_t warp = warp_id(), lane = lane_id();
  const int kblock = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int group = p.nheads / p.nheads_kv;
  const int k0 = kblock * BN;
  const int k1 = min(k0 + BN, p.seqlen_k);

  // Query rows that see any key of [k0, k1).
  const long long off = (long long)p.seqlen_k - p.seqlen_q;
  const long long kInf = 1ll << 40;
  const long long rb = p.causal ? 0 : (p.window_right >= 0 ? p.window_right : kInf);
  const long long lb = p.window_left >= 0 ? p.window_left : kInf;
  long long imin = (long long)k0 - off - rb;
  long long imax = (long long)(k1 - 1) - off + lb;
  if (imin < 0) imin = 0;
  if (imax > (long long)p.seqlen_q - 1) imax = (long long)p.seqlen_q - 1;
  const int qb_lo = imax >= imin ? (int)(imin / BM) : 0;
  const int nqb = imax >= imin ? (int)(imax / BM) - qb_lo + 1 : 0;
  const int nt = nqb * group;  // tiles: (head in group) x (query tile)

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NBAR; ++i) {
      const bool many = i == C::B_PREADY || i == C::B_DSREADY || i == C::B_DQFREE;
      mbar_init(bar(i), many ? 128 : 1);
    }
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem0 + C::OFF_TMEMPTR, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nt > 0) {
      mbar_arrive_expect_tx(bar(C::B_KV), 2 * C::KV_BYTES);
      for (int bx = 0; bx < C::NBOX; ++bx) {
        tma_load_4d(smem0 + C::OFF_K + bx * (BN * 128), &tm_k, bar(C::B_KV), bx * 64, kvh, k0, b);
        tma_load_4d(smem0 + C::OFF_V + bx * (BN * 128), &tm_v, bar(C::B_KV), bx * 64, kvh, k0, b);
      }
      for (int t = 0; t < nt; ++t) {
        const int st = t & 1, n = t >> 1;
        if (n > 0 && !mbar_wait(bar(C::B_EMPTY + st), (n - 1) & 1)) break;
        const int h = kvh * group + t / nqb;
        const int q0 = (qb_lo + t % nqb) * BM;
        const int row = (b * p.nheads + h);
        mbar_arrive_expect_tx(bar(C::B_QFULL + st), C::Q_BYTES + BM * 4);
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_load_4d(smem0 + C::OFF_Q + st * C::Q_BYTES + bx * (BM * 128), &tm_q,
                      bar(C::B_QFULL + st), bx * 64, h, q0, b);
        tma_load_2d(smem0 + C::OFF_LSE + st * BM * 4, &tm_lse2, bar(C::B_QFULL + st), q0, row);
        mbar_arrive_expect_tx(bar(C::B_DOFULL + st), C::Q_BYTES + BM * 4);
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_load_4d(smem0 + C::OFF_DO + st * C::Q_BYTES + bx * (BM * 128), &tm_do,
                      bar(C::B_DOFULL + st), bx * 64, h, q0, b);
        tma_load_2d(smem0 + C::OFF_DVEC + st * BM * 4, &tm_dvec, bar(C::B_DOFULL + st), q0, row);
      }
      for (int t = nt - 2 < 0 ? 0 : nt - 2; t < nt; ++t) {
        const int st = t & 1, n = t >> 1;
        if (!mbar_wait(bar(C::B_QFULL + st), n & 1)) break;
        if (!mbar_wait(bar(C::B_DOFULL + st), n & 1)) break;
      }
      mbar_wait(bar(C::B_KV), 0);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nt > 0) {
      constexpr uint32_t idesc_s = idesc_f16(BN, BM, C::FP16, false, false);
      constexpr uint32_t idesc_acc = idesc_f16(BN, D, C::FP16, false, true);
      constexpr uint32_t idesc_dq =
          C::DQT ? idesc_f16(D, BM, C::FP16, true, true) : idesc_f16(BM, D, C::FP16, true, true);
      const uint32_t k_base = smem0 + C::OFF_K, v_base = smem0 + C::OFF_V;
      const uint32_t ds_base = smem0 + C::OFF_DS;
      bool ok = mbar_wait(bar(C::B_KV), 0);
      for (int t = 0; ok && t < nt; ++t) {
        const int st = t & 1, ph = (t >> 1) & 1;
        const uint32_t q_base = smem0 + C::OFF_Q + st * C::Q_BYTES;
        const uint32_t do_base = smem0 + C::OFF_DO + st * C::Q_BYTES;
        if (!mbar_wait(bar(C::B_QFULL + st), ph)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {  // S^T = K Q^T
          const int bx = kk / 4, w = kk % 4;
          mma_ss(tmem + C::TM_S, sdesc_sw128(k_base + bx * (BN * 128) + w * 32, 16, 1024),
                 sdesc_sw128(q_base + bx * (BM * 128) + w * 32, 16, 1024), idesc_s, kk > 0);
        }
        mma_commit(bar(C::B_SFULL));
        if (!mbar_wait(bar(C::B_DOFULL + st), ph)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {  // dP^T = V dO^T
          const int bx = kk / 4, w = kk % 4;
          mma_ss(tmem + C::TM_DP, sdesc_sw128(v_base + bx * (BN * 128) + w * 32, 16, 1024),
                 sdesc_sw128(do_base + bx * (BM * 128) + w * 32, 16, 1024), idesc_s, kk > 0);
        }
        mma_commit(bar(C::B_DPFULL));
        if (!mbar_wait(bar(C::B_PREADY), t & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)  // dV += P^T dO
          mma_ts(tmem + C::TM_DV, tmem + C::TM_S + kk * 8,
                 sdesc_sw128(do_base + kk * 2048, BM * 128, 1024), idesc_acc, (t > 0 || kk > 0));
        if (!mbar_wait(bar(C::B_DSREADY), t & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)  // dK += dS^T Q
          mma_ts(tmem + C::TM_DK, tmem + C::TM_DP + kk * 8,
                 sdesc_sw128(q_base + kk * 2048, BM * 128, 1024), idesc_acc, (t > 0 || kk > 0));
        if (t > 0 && !mbar_wait(bar(C::B_DQFREE), (t - 1) & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          if constexpr (C::DQT)  // dQ^T = K^T dS^T: both operands MN-major
            mma_ss(tmem + C::TM_DQ, sdesc_sw128(k_base + kk * 2048, BN * 128, 1024),
                   sdesc_sw128(ds_base + kk * 2048, BN * 128, 1024), idesc_dq, kk > 0);
          else  // dQ = dS K
            mma_ss(tmem + C::TM_DQ, sdesc_sw128(ds_base + kk * 2048, BN * 128, 1024),
                   sdesc_sw128(k_base + kk * 2048, BN * 128, 1024), idesc_dq, kk > 0);
        }
        mma_commit(bar(C::B_DQFULL));
        mma_commit(bar(C::B_DSFREE));
        mma_commit(bar(C::B_EMPTY + st));
      }
      if (ok) mma_commit(bar(C::B_DONE));
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ P / dS
    const int r = (int)threadIdx.x;  // key row within the tile == TMEM lane
    const long long j = (long long)k0 + r;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    bool ok = true;
    for (int t = 0; t < nt; ++t) {
      const int st = t & 1, ph = (t >> 1) & 1;
      const int q0 = (qb_lo + t % nqb) * BM;
      if (!mbar_wait_warp(bar(C::B_SFULL), t & 1)) { ok = false; break; }
      if (!mbar_wait_warp(bar(C::B_QFULL + st), ph)) { ok = false; break; }
      tc_fence_after();
      float pr[BM];
#pragma unroll
      for (int c = 0; c < BM; c += 32) {
        uint32_t raw[32];
        tmem_ld32(tmem + lane_base + C::TM_S + c, raw);
#pragma unroll
        for (int e = 0; e < 32; ++e) pr[c + e] = __uint_as_float(raw[e]);
      }
      tmem_ld_wait();
      const float* lse_t = lse_s + st * BM;
      // Whole tile visible (query rows past seqlen_q have LSE2 = +inf, so P = 0).
      const bool full = ((long long)k0 + BN <= p.seqlen_k) &&
                        ((long long)k0 + BN - 1 <= (long long)q0 + off + rb) &&
                        ((long long)k0 >= (long long)(q0 + BM - 1) + off - lb);
#pragma unroll
      for (int c = 0; c < BM; ++c) {
        float v = ex2(fmaf(pr[c], p.scale_log2, -lse_t[c]));
        if (!full) {
          const long long i = (long long)q0 + c;
          if (j >= p.seqlen_k || j > i + off + rb || j < i + off - lb) v = 0.f;
        }
        pr[c] = v;
      }
      {
        uint32_t w[BM / 2];
#pragma unroll
        for (int c = 0; c < BM; c += 2) w[c / 2] = pack2<C::FP16>(pr[c], pr[c + 1]);
#pragma unroll
        for (int c = 0; c < BM / 2; c += 16) {
          uint32_t chunk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) chunk[e] = w[c + e];
          tmem_st16(tmem + lane_base + C::TM_S + c, chunk);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(C::B_PREADY));
      if (!mbar_wait_warp(bar(C::B_DPFULL), t & 1)) { ok = false; break; }
      if (!mbar_wait_warp(bar(C::B_DOFULL + st), ph)) { ok = false; break; }
      tc_fence_after();
      const float* dvec_t = dvec_s + st * BM;
#pragma unroll
      for (int c = 0; c < BM; c += 32) {
        uint32_t raw[32];
        tmem_ld32(tmem + lane_base + C::TM_DP + c, raw);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) pr[c + e] = pr[c + e] * (__uint_as_float(raw[e]) - dvec_t[c + e]);
      }
      // dS smem tile is free once the previous tile's dQ MMA has read it.
      if (t > 0 && !mbar_wait_warp(bar(C::B_DSFREE), (t - 1) & 1)) { ok = false; break; }
      {
        uint32_t w[BM / 2];
#pragma unroll
        for (int c = 0; c < BM; c += 2) w[c / 2] = pack2<C::FP16>(pr[c], pr[c + 1]);
#pragma unroll
        for (int c = 0; c < BM / 2; c += 16) {
          uint32_t chunk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) chunk[e] = w[c + e];
          tmem_st16(tmem + lane_base + C::TM_DP + c, chunk);
        }
        // dS as [key row][query] with 128-byte swizzle, 64 queries per box.
        const uint32_t row_addr = smem0 + C::OFF_DS + r * 128;
#pragma unroll
        for (int c8 = 0; c8 < BM / 8; ++c8) {
          const int bx = c8 / 8, chunk = (c8 % 8) ^ (r & 7);
          st_shared_v4(row_addr + bx * (BN * 128) + chunk * 16, w[4 * c8], w[4 * c8 + 1],
                       w[4 * c8 + 2], w[4 * c8 + 3]);
        }
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(C::B_DSREADY));
    }
    // ------------------------------------------------------------ epilogue
    if (ok && nt > 0) ok = mbar_wait_warp(bar(C::B_DONE), 0);
    if (ok) {
      tc_fence_after();
      // dK (x scale) staged in the Q slots, dV in the dO slots.
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t src = tmem + lane_base + (which == 0 ? C::TM_DK : C::TM_DV);
        const uint32_t row_addr = smem0 + (which == 0 ? C::OFF_Q : C::OFF_DO) + r * 128;
        const float mul = which == 0 ? p.softmax_scale : 1.f;
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t raw[32];
          if (nt > 0) {
            tmem_ld32(src + c, raw);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) raw[e] = 0u;
          }
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[e] = pack2<C::FP16>(__uint_as_float(raw[2 * e]) * mul, __uint_as_float(raw[2 * e + 1]) * mul);
          const int bx = c / 64, chunk0 = (c % 64) / 8;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int chunk = (chunk0 + q4) ^ (r & 7);
            st_shared_v4(row_addr + bx * (BN * 128) + chunk * 16, w[4 * q4], w[4 * q4 + 1],
                         w[4 * q4 + 2], w[4 * q4 + 3]);
          }
        }
      }
      fence_proxy_async_smem();
    }
    tc_fence_before();
    named_bar_sync(1, 128);
    if (ok && threadIdx.x == 0) {
      for (int bx = 0; bx < C::NBOX; ++bx) {
        tma_store_4d(&tm_dk, smem0 + C::OFF_Q + bx * (BN * 128), bx * 64, kvh, k0, b);
        tma_store_4d(&tm_dv, smem0 + C::OFF_DO + bx * (BN * 128), bx * 64, kvh, k0, b);
      }
      bulk_commit_group();
      bulk_wait_group_all();
    }
  } else {
    // ------------------------------------------------------------ dQ readout (warps 4-7)
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int r = (int)((warp & 3) * 32 + lane);  // TMEM lane
    for (int t = 0; t < nt; ++t) {
      const int h = kvh * group + t / nqb;
      const int q0 = (qb_lo + t % nqb) * BM;
      if (!mbar_wait_warp(bar(C::B_DQFULL), t & 1)) break;
      tc_fence_after();
      if constexpr (C::DQT) {
        // lane = head-dim column r, columns = query rows q0..q0+BM
        float vals[BM];
#pragma unroll
        for (int c = 0; c < BM; c += 32) {
          uint32_t raw[32];
          tmem_ld32(tmem + lane_base + C::TM_DQ + c, raw);
#pragma unroll
          for (int e = 0; e < 32; ++e) vals[c + e] = __uint_as_float(raw[e]);
        }
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(bar(C::B_DQFREE));
        float* dst = p.dq_acc + (((size_t)b * p.seqlen_q + q0) * p.nheads + h) * D + r;
        const size_t row_stride = (size_t)p.nheads * D;
#pragma unroll 8
        for (int c = 0; c < BM; ++c)
          if (q0 + c < p.seqlen_q) atomicAdd(dst + c * row_stride, vals[c]);
      } else {
        // lane = query row q0 + r, columns = head-dim
        float vals[D];
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t raw[32];
          tmem_ld32(tmem + lane_base + C::TM_DQ + c, raw);
#pragma unroll
          for (int e = 0; e < 32; ++e) vals[c + e] = __uint_as_float(raw[e]);
        }
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(bar(C::B_DQFREE));
        if (q0 + r < p.seqlen_q) {
          float4* dst = reinterpret_cast<float4*>(
              p.dq_acc + (((size_t)b * p.seqlen_q + q0 + r) * p.nheads + h) * D);
#pragma unroll
          for (int c = 0; c < D / 4; ++c)
            atomicAdd(dst + c, make_float4(vals[4 * c], vals[4 * c + 1], vals[4 * c + 2], vals[4 * c + 3]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace attn
