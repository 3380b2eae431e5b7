// bwd256_kernel.cuh - exact attention backward pass for head dimension 256
// on sm_100a.
//
// The method is the one of bwd_kernel.cuh (score tiles recomputed from Q, K
// and the saved log-sum-exp, "FlashAttention ... transformer optimization",
// item 2; FlashAttention-2 supports d = 256 in the backward, "FlashAttention
// 四代演进", hardware / dtype limits).  What changes at d = 256 is the
// budget: one 128-key tile's fp32 dK and dV take all 512 tensor-memory
// columns, and its K and V tiles 128 KB of shared memory.  So the gradients
// come from three kernels, each holding one accumulator in tensor memory and
// recomputing the score tiles it needs:
//
//   attn_bwd256_kv_kernel<C<.., false>>  dV = P^T dO          S^T = K Q^T
//   attn_bwd256_kv_kernel<C<.., true>>   dK = scale dS^T Q    S^T, dP^T = V dO^T
//   attn_bwd256_q_kernel                 dQ acc += dS K       S = Q K^T, dP = dO V^T
//
// with P = exp2(S * scale * log2 e - LSE2) and dS = P o (dP - Dvec) as in the
// main kernel (LSE2 and Dvec are the fp32 rows bwd_preprocess writes).
// Eight products of a tile pair instead of five; each kernel stays within
// the tensor-memory and shared-memory budgets with its MMAs double-buffered.
// The first two are key-stationary (one CTA per (batch, kv head, 128-key
// tile), walking the 64-query tiles of every query head of its group); the
// third is query-stationary (one CTA per (batch, head, 128-query tile),
// walking the visible 64-key tiles), so it owns its dQ rows and adds them to
// the fp32 accumulator that bwd_convert scales and rounds.  The outputs
// leave the kernels from registers (16-byte stores per thread), one row per
// thread.
#pragma once

#include "bwd_kernel.cuh"
#include "sm100.cuh"

namespace attn {

// ------------------------------------------------------------ key-stationary
// Roles (320 threads): warp 8 TMA producer (K, and V for dK; Q and dO per
// query tile through rings of their own), warp 9 tensor-memory allocation and
// MMA issue, warps 0-7 two per lane quadrant (one thread per key row), each
// owning 32 of the tile's 64 query columns.
template <bool FP16_, bool DK_>
struct Bwd256KvCfg {
  static constexpr bool FP16 = FP16_, DK = DK_;
  static constexpr int D = 256, BN = 128, BM = 64, NBUF = 2, NBOX = D / 64;
  static constexpr int HW = BM / 2;  // query columns per compute warp
  // dV: Q is read only by S^T, dO only by the dV product; dK: Q by S^T and
  // the dK product, dO only by dP^T (issued a tile ahead of its use).
  static constexpr int QSTAGES = 2, DOSTAGES = DK ? 1 : 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_BYTES;  // dK only
  static constexpr int OFF_Q = OFF_V + (DK ? KV_BYTES : 0);
  static constexpr int OFF_DO = OFF_Q + QSTAGES * Q_BYTES;
  static constexpr int OFF_BAR = OFF_DO + DOSTAGES * Q_BYTES;
  static constexpr int B_KV = 0;
  static constexpr int B_QFULL = 1;
  static constexpr int B_DOFULL = B_QFULL + QSTAGES;
  static constexpr int B_QEMPTY = B_DOFULL + DOSTAGES;
  static constexpr int B_DOEMPTY = B_QEMPTY + QSTAGES;
  static constexpr int B_SFULL = B_DOEMPTY + DOSTAGES;  // per buffer
  static constexpr int B_DPFULL = B_SFULL + NBUF;        // per buffer (dK)
  static constexpr int B_XREADY = B_DPFULL + NBUF;       // P^T / dS^T in TMEM: 256 arrivals
  static constexpr int B_DONE = B_XREADY + NBUF;
  static constexpr int B_FLUSH = B_DONE + 1;  // every MMA of the CTA complete
  static constexpr int NBAR = B_FLUSH + 1;
  static constexpr int OFF_TMEMPTR = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_TMEMPTR + 16 + 1024;
  // tensor memory: the accumulator (dV or dK), then per buffer an S^T block
  // (and for dK a dP^T block) of BM fp32 columns
  static constexpr int TM_ACC = 0, TM_S = D, TM_DP = D + NBUF * BM;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 320;
  static_assert(TM_DP + (DK ? NBUF * BM : 0) <= TMEM_COLS, "tensor memory");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// `out`: dV (DK false) or dK (DK true), (batch, seqlen_k, nheads_kv, 256) in
// the input dtype, or float32 sums to add into when p.acc_f32.
template <class C, bool ALIBI>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_bwd256_kv_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_do, const BwdParams pin,
                          void* out) {
  constexpr int D = C::D, BN = C::BN, BM = C::BM, NBUF = C::NBUF, HW = C::HW;
  constexpr int QS = C::QSTAGES, DS = C::DOSTAGES;
  constexpr bool DK = C::DK;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem0 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem0 - smem_addr(smem_raw));
  auto bar = [&](int i) -> uint32_t { return smem0 + C::OFF_BAR + 8u * i; };
  volatile uint32_t* tmem_ptr_slot = reinterpret_cast<volatile uint32_t*>(smem_gen + C::OFF_TMEMPTR);
  const uint32_t warp = warp_id(), lane = lane_id();

  // key tile 0 is seen by the most queries under a causal mask: rank order
  const UnitOrder uo = grouped_lpt((int)blockIdx.x, pin.num_kblocks, pin.batch * pin.nheads_kv,
                                   pin.sched_group);
  const int kblock = uo.rank, kvh = uo.head % pin.nheads_kv, b = uo.head / pin.nheads_kv;
  const SeqSpan sq = seq_span(pin.cu_q, pin.cu_k, pin.total_q, pin.total_k, b, pin.seqlen_q,
                              pin.seqlen_k);
  BwdParams p = pin;  // lengths of this block's sequence
  p.seqlen_q = sq.len_q;
  p.seqlen_k = sq.len_k;
  const int group = p.nheads / p.nheads_kv;
  const int k0 = kblock * BN;
  if (k0 >= p.seqlen_k) return;  // past a packed sequence: nothing to do
  const int k1 = min(k0 + BN, p.seqlen_k);
  const long long prow0 = p.cu_q ? packed_row0(sq.q_row0, b) : 0;

  // query rows that see any key of [k0, k1)
  const long long off = (long long)p.seqlen_k - p.seqlen_q + p.pos_offset;
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

  auto tile_coords = [&](int t, int& h, int& q0) {
    h = kvh * group + t / nqb;
    q0 = (qb_lo + t % nqb) * BM;
  };
  auto load_q = [&](int t) -> bool {
    const int slot = t % QS, n = t / QS;
    if (n > 0 && !mbar_wait(bar(C::B_QEMPTY + slot), (n - 1) & 1)) return false;
    int h, q0;
    tile_coords(t, h, q0);
    mbar_arrive_expect_tx(bar(C::B_QFULL + slot), C::Q_BYTES);
    for (int bx = 0; bx < C::NBOX; ++bx)
      tma_load_4d(smem0 + C::OFF_Q + slot * C::Q_BYTES + bx * (BM * 128), &tm_q,
                  bar(C::B_QFULL + slot), bx * 64, h, sq.q_row0 + q0, sq.tma_b);
    return true;
  };
  auto load_do = [&](int t) -> bool {
    const int slot = t % DS, n = t / DS;
    if (n > 0 && !mbar_wait(bar(C::B_DOEMPTY + slot), (n - 1) & 1)) return false;
    int h, q0;
    tile_coords(t, h, q0);
    mbar_arrive_expect_tx(bar(C::B_DOFULL + slot), C::Q_BYTES);
    for (int bx = 0; bx < C::NBOX; ++bx)
      tma_load_4d(smem0 + C::OFF_DO + slot * C::Q_BYTES + bx * (BM * 128), &tm_do,
                  bar(C::B_DOFULL + slot), bx * 64, h, sq.q_row0 + q0, sq.tma_b);
    return true;
  };

  if (warp == 8 && lane == 0) {
    for (int i = 0; i < C::NBAR; ++i)
      mbar_init(bar(i), (i >= C::B_XREADY && i < C::B_XREADY + NBUF) ? 256u : 1u);
    fence_barrier_init();
    fence_proxy_async_smem();
    if (nt > 0) {
      mbar_arrive_expect_tx(bar(C::B_KV), (DK ? 2 : 1) * C::KV_BYTES);
      for (int bx = 0; bx < C::NBOX; ++bx) {
        tma_load_4d(smem0 + C::OFF_K + bx * (BN * 128), &tm_k, bar(C::B_KV), bx * 64, kvh,
                    sq.k_row0 + k0, sq.tma_b);
        if constexpr (DK)
          tma_load_4d(smem0 + C::OFF_V + bx * (BN * 128), &tm_v, bar(C::B_KV), bx * 64, kvh,
                      sq.k_row0 + k0, sq.tma_b);
      }
      load_q(0);
      load_do(0);
    }
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
      for (int t = 1; t < nt; ++t)
        if (!load_q(t) || !load_do(t)) break;
      for (int t = nt - QS < 0 ? 0 : nt - QS; t < nt; ++t)
        if (!mbar_wait(bar(C::B_QFULL + t % QS), (t / QS) & 1)) break;
      for (int t = nt - DS < 0 ? 0 : nt - DS; t < nt; ++t)
        if (!mbar_wait(bar(C::B_DOFULL + t % DS), (t / DS) & 1)) break;
      mbar_wait(bar(C::B_KV), 0);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (nt > 0) {
      constexpr uint32_t idesc_s = idesc_f16(BN, BM, C::FP16, false, false);
      constexpr uint32_t idesc_acc = idesc_f16(BN, D, C::FP16, false, true);
      const uint64_t k_kdesc = sdesc_sw128(smem0 + C::OFF_K, 16, 1024);
      const uint64_t v_kdesc = sdesc_sw128(smem0 + C::OFF_V, 16, 1024);
      // S^T_u = K Q_u^T into the S block of buffer u % NBUF
      auto issue_s = [&](int u) -> bool {
        const int slot = u % QS, bf = u % NBUF;
        const uint64_t q_desc = sdesc_sw128(smem0 + C::OFF_Q + slot * C::Q_BYTES, 16, 1024);
        if (!mbar_wait_warp(bar(C::B_QFULL + slot), (u / QS) & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int bx = kk / 4, w = kk % 4;
          mma_ss_warp(tmem + C::TM_S + bf * BM, desc_at(k_kdesc, bx * (BN * 128) + w * 32),
                      desc_at(q_desc, bx * (BM * 128) + w * 32), idesc_s, kk > 0);
        }
        mma_commit_warp(bar(C::B_SFULL + bf));
        if constexpr (!DK) mma_commit_warp(bar(C::B_QEMPTY + slot));
        return true;
      };
      // dP^T_u = V dO_u^T into the dP block of buffer u % NBUF (dK)
      auto issue_dp = [&](int u) -> bool {
        const int slot = u % DS, bf = u % NBUF;
        const uint64_t do_desc = sdesc_sw128(smem0 + C::OFF_DO + slot * C::Q_BYTES, 16, 1024);
        if (!mbar_wait_warp(bar(C::B_DOFULL + slot), (u / DS) & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int bx = kk / 4, w = kk % 4;
          mma_ss_warp(tmem + C::TM_DP + bf * BM, desc_at(v_kdesc, bx * (BN * 128) + w * 32),
                      desc_at(do_desc, bx * (BM * 128) + w * 32), idesc_s, kk > 0);
        }
        mma_commit_warp(bar(C::B_DPFULL + bf));
        mma_commit_warp(bar(C::B_DOEMPTY + slot));
        return true;
      };
      // acc += X^T B: X^T = P^T (dV, B = dO) or dS^T (dK, B = Q), 16-bit in
      // the first columns of each half of the tile's S block; B MN-major.
      auto issue_grad = [&](int t) -> bool {
        const int bf = t % NBUF, use = t / NBUF;
        const uint32_t b_base = DK ? smem0 + C::OFF_Q + (t % QS) * C::Q_BYTES
                                   : smem0 + C::OFF_DO + (t % DS) * C::Q_BYTES;
        const uint64_t b_mn = sdesc_sw128(b_base, BM * 128, 1024);
        if (!mbar_wait_warp(bar(C::B_XREADY + bf), use & 1)) return false;
        // dV: nothing else waits for the dO slot (the compute warps do not
        // read it); dK: issue_s(t) waited for the Q slot
        if (!DK && !mbar_wait_warp(bar(C::B_DOFULL + t % DS), (t / DS) & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk) {
          const int half = kk / (HW / 16), part = kk % (HW / 16);
          mma_ts_warp(tmem + C::TM_ACC, tmem + C::TM_S + bf * BM + half * HW + part * 8,
                      desc_at(b_mn, kk * 2048), idesc_acc, (t > 0 || kk > 0));
        }
        if constexpr (DK)
          mma_commit_warp(bar(C::B_QEMPTY + t % QS));
        else
          mma_commit_warp(bar(C::B_DOEMPTY + t % DS));
        return true;
      };
      // Tile t+1's S^T (and dP^T) go in around tile t's accumulation, so the
      // tensor pipe works on one tile while the compute warps exponentiate
      // the other.
      bool ok = mbar_wait_warp(bar(C::B_KV), 0) && issue_s(0) && (!DK || issue_dp(0));
      for (int t = 0; ok && t < nt; ++t) {
        const bool more = t + 1 < nt;
        if (more && !issue_s(t + 1)) { ok = false; break; }
        if (!issue_grad(t)) { ok = false; break; }
        if (DK && more && !issue_dp(t + 1)) { ok = false; break; }
      }
      if (ok) mma_commit_warp(bar(C::B_DONE));
    }
  } else {
    // ------------------------------------------------------------ P, dS
    const int quad = (int)(warp & 3), half = (int)(warp >> 2);
    const int r = quad * 32 + (int)lane;  // key row within the tile == TMEM lane
    const int c0 = half * HW;             // first query column of this warp
    const long long j = (long long)k0 + r;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
    bool ok = true;
    for (int t = 0; t < nt; ++t) {
      const int bf = t % NBUF, use = t / NBUF;
      int hq, q0;
      tile_coords(t, hq, q0);
      const int qa = q0 + c0;
      // LSE2 (and Dvec) of this warp's 32 query columns: the same addresses
      // in every lane (broadcast loads), issued before the wait.  Padding
      // rows hold LSE2 = +inf, so their P is 0.
      const size_t srow = (size_t)(p.cu_q ? hq : b * p.nheads + hq) * p.nq_pad + prow0 + qa;
      float lse[HW];
      [[maybe_unused]] float dv[HW];
#pragma unroll
      for (int c = 0; c < HW; c += 4) {
        const float4 l4 = __ldg(reinterpret_cast<const float4*>(p.lse2 + srow + c));
        lse[c] = l4.x, lse[c + 1] = l4.y, lse[c + 2] = l4.z, lse[c + 3] = l4.w;
        if constexpr (DK) {
          const float4 d4 = __ldg(reinterpret_cast<const float4*>(p.dvec + srow + c));
          dv[c] = d4.x, dv[c + 1] = d4.y, dv[c + 2] = d4.z, dv[c + 3] = d4.w;
        }
      }
      if (!mbar_wait_warp(bar(C::B_SFULL + bf), use & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t s_tmem = tmem + lane_base + C::TM_S + bf * BM + c0;
      float pr[HW];
      {
        uint32_t raw[32];
        tmem_ld32(s_tmem, raw);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < HW; ++c) pr[c] = __uint_as_float(raw[c]);
      }
      const bool full = ((long long)k0 + BN <= p.seqlen_k) &&
                        ((long long)k0 + BN - 1 <= (long long)qa + off + rb) &&
                        ((long long)k0 >= (long long)(qa + HW - 1) + off - lb);
      const float bk = ALIBI ? -p.alibi[hq] * 1.4426950408889634f : 0.f;
      const float bd = ALIBI ? (float)(j - off - qa) : 0.f;
#pragma unroll
      for (int c = 0; c < HW; c += 2) {
        float a0, a1;
        f2_unpack(f2_fma(f2_pack(pr[c], pr[c + 1]), scale2, f2_pack(-lse[c], -lse[c + 1])), a0,
                  a1);
        if constexpr (ALIBI) {
          a0 = fmaf(fabsf((float)c - bd), bk, a0);
          a1 = fmaf(fabsf((float)(c + 1) - bd), bk, a1);
        }
        pr[c] = ex2(a0);
        pr[c + 1] = ex2(a1);
      }
      if (!full) {
#pragma unroll
        for (int c = 0; c < HW; ++c) {
          const long long i = (long long)qa + c;
          if (j >= p.seqlen_k || j > i + off + rb || j < i + off - lb) pr[c] = 0.f;
        }
      }
      if constexpr (DK) {
        if (!mbar_wait_warp(bar(C::B_DPFULL + bf), use & 1)) { ok = false; break; }
        tc_fence_after();
        uint32_t raw[32];
        tmem_ld32(tmem + lane_base + C::TM_DP + bf * BM + c0, raw);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < HW; c += 2)
          f2_unpack(f2_mul(f2_pack(pr[c], pr[c + 1]),
                           f2_add(f2_pack(__uint_as_float(raw[c]), __uint_as_float(raw[c + 1])),
                                  f2_pack(-dv[c], -dv[c + 1]))),
                    pr[c], pr[c + 1]);
      }
      // P^T (dV) or dS^T (dK), 16-bit, over this half's first score columns
      // (already read): the A operand of the accumulation
      uint32_t w[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) w[e] = pack2<C::FP16>(pr[2 * e], pr[2 * e + 1]);
      tmem_st16(s_tmem, w);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(C::B_XREADY + bf));
    }
    // ------------------------------------------------------------ epilogue
    // This warp's key rows x head-dim columns [half * 128, half * 128 + 128)
    // of the accumulator, (x scale for dK) straight to global memory.
    if (ok && nt > 0) ok = mbar_wait_warp(bar(C::B_DONE), 0);
    if (ok && !(p.acc_f32 && nt == 0)) {
      tc_fence_after();
      const float mul = DK ? p.softmax_scale : 1.f;
      const bool row_ok = j < p.seqlen_k;
      const size_t orow =
          (((size_t)sq.tma_b * pin.seqlen_k + sq.k_row0 + (size_t)j) * p.nheads_kv + kvh) * D;
#pragma unroll 1
      for (int c = half * (D / 2); c < (half + 1) * (D / 2); c += 32) {
        uint32_t raw[32];
        if (nt > 0) {
          tmem_ld32(tmem + lane_base + C::TM_ACC + c, raw);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) raw[e] = 0u;
        }
        if (!row_ok) continue;
        if (p.acc_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + orow + c);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float4 a = dst[e];
            a.x += __uint_as_float(raw[4 * e]) * mul;
            a.y += __uint_as_float(raw[4 * e + 1]) * mul;
            a.z += __uint_as_float(raw[4 * e + 2]) * mul;
            a.w += __uint_as_float(raw[4 * e + 3]) * mul;
            dst[e] = a;
          }
        } else {
          uint32_t wv[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            wv[e] = pack2<C::FP16>(__uint_as_float(raw[2 * e]) * mul,
                                   __uint_as_float(raw[2 * e + 1]) * mul);
          store_row32(static_cast<uint16_t*>(out) + orow + c, wv);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    // every MMA this warp issued has completed (also on a path that gave
    // up early) before the tensor memory is released
    if (nt > 0) {
      mma_commit_warp(bar(C::B_FLUSH));
      mbar_wait_warp(bar(C::B_FLUSH), 0);
    }
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------ query-stationary
// Roles (320 threads): warp 8 TMA producer (Q and dO once; K and V per 64-key
// tile through rings of their own), warp 9 tensor-memory allocation and MMA
// issue, warps 0-7 two per lane quadrant (one thread per query row), each
// owning 32 of the tile's 64 key columns.
template <bool FP16_>
struct Bwd256QCfg {
  static constexpr bool FP16 = FP16_;
  static constexpr int D = 256, BM = 128, BN = 64, NBUF = 2, NBOX = D / 64;
  static constexpr int HW = BN / 2;  // key columns per compute warp
  // K_j is read by S_j and by the dQ product of tile j (issued a tile
  // later), V_j only by dP_j.
  static constexpr int KSTAGES = 2, VSTAGES = 1;
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = OFF_Q + Q_BYTES;
  static constexpr int OFF_K = OFF_DO + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KSTAGES * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + VSTAGES * KV_BYTES;
  static constexpr int B_QDO = 0;
  static constexpr int B_KFULL = 1;
  static constexpr int B_KEMPTY = B_KFULL + KSTAGES;
  static constexpr int B_VFULL = B_KEMPTY + KSTAGES;
  static constexpr int B_VEMPTY = B_VFULL + VSTAGES;
  static constexpr int B_SFULL = B_VEMPTY + VSTAGES;  // per buffer
  static constexpr int B_DPFULL = B_SFULL + NBUF;      // per buffer
  static constexpr int B_DSREADY = B_DPFULL + NBUF;    // dS in TMEM: 256 arrivals
  static constexpr int B_DONE = B_DSREADY + NBUF;
  static constexpr int B_FLUSH = B_DONE + 1;  // every MMA of the CTA complete
  static constexpr int NBAR = B_FLUSH + 1;
  static constexpr int OFF_TMEMPTR = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_TMEMPTR + 16 + 1024;
  // tensor memory: per buffer an S block and a dP block of BN fp32 columns,
  // then the dQ accumulator (D columns)
  static constexpr int TM_S = 0, TM_DP = NBUF * BN, TM_DQ = 2 * NBUF * BN;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 320;
  static_assert(TM_DQ + D <= TMEM_COLS, "tensor memory");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <class C, bool ALIBI>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_bwd256_q_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_do, const BwdParams pin) {
  constexpr int D = C::D, BN = C::BN, BM = C::BM, NBUF = C::NBUF, HW = C::HW;
  constexpr int KS = C::KSTAGES, VS = C::VSTAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem0 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem0 - smem_addr(smem_raw));
  auto bar = [&](int i) -> uint32_t { return smem0 + C::OFF_BAR + 8u * i; };
  volatile uint32_t* tmem_ptr_slot = reinterpret_cast<volatile uint32_t*>(smem_gen + C::OFF_TMEMPTR);
  const uint32_t warp = warp_id(), lane = lane_id();

  // later query tiles see more keys under a causal mask: heaviest first
  const UnitOrder uo = grouped_lpt((int)blockIdx.x, pin.num_qblocks, pin.batch * pin.nheads,
                                   pin.sched_group);
  const int qt = pin.num_qblocks - 1 - uo.rank;
  const int h = uo.head % pin.nheads, b = uo.head / pin.nheads;
  const SeqSpan sq = seq_span(pin.cu_q, pin.cu_k, pin.total_q, pin.total_k, b, pin.seqlen_q,
                              pin.seqlen_k);
  BwdParams p = pin;
  p.seqlen_q = sq.len_q;
  p.seqlen_k = sq.len_k;
  const int q0 = qt * BM;
  if (q0 >= p.seqlen_q) return;  // past a packed sequence: nothing to do
  const int kvh = h / (p.nheads / p.nheads_kv);
  const long long prow0 = p.cu_q ? packed_row0(sq.q_row0, b) : 0;

  // key tiles [lo, hi) seen by rows [q0, q1)
  const int q1 = min(q0 + BM, p.seqlen_q);
  const long long off = (long long)p.seqlen_k - p.seqlen_q + p.pos_offset;
  const long long kInf = 1ll << 40;
  const long long rb = p.causal ? 0 : (p.window_right >= 0 ? p.window_right : kInf);
  const long long lb = p.window_left >= 0 ? p.window_left : kInf;
  long long jmin = (long long)q0 + off - lb, jmax = (long long)(q1 - 1) + off + rb;
  if (jmin < 0) jmin = 0;
  if (jmax > (long long)p.seqlen_k - 1) jmax = (long long)p.seqlen_k - 1;
  const int lo = jmax >= jmin ? (int)(jmin / BN) : 0;
  const int nt = jmax >= jmin ? (int)(jmax / BN) - lo + 1 : 0;

  auto load_k = [&](int n) -> bool {  // key tile lo + n
    const int slot = n % KS, u = n / KS;
    if (u > 0 && !mbar_wait(bar(C::B_KEMPTY + slot), (u - 1) & 1)) return false;
    mbar_arrive_expect_tx(bar(C::B_KFULL + slot), C::KV_BYTES);
    for (int bx = 0; bx < C::NBOX; ++bx)
      tma_load_4d(smem0 + C::OFF_K + slot * C::KV_BYTES + bx * (BN * 128), &tm_k,
                  bar(C::B_KFULL + slot), bx * 64, kvh, sq.k_row0 + (lo + n) * BN, sq.tma_b);
    return true;
  };
  auto load_v = [&](int n) -> bool {
    const int slot = n % VS, u = n / VS;
    if (u > 0 && !mbar_wait(bar(C::B_VEMPTY + slot), (u - 1) & 1)) return false;
    mbar_arrive_expect_tx(bar(C::B_VFULL + slot), C::KV_BYTES);
    for (int bx = 0; bx < C::NBOX; ++bx)
      tma_load_4d(smem0 + C::OFF_V + slot * C::KV_BYTES + bx * (BN * 128), &tm_v,
                  bar(C::B_VFULL + slot), bx * 64, kvh, sq.k_row0 + (lo + n) * BN, sq.tma_b);
    return true;
  };

  if (warp == 8 && lane == 0) {
    for (int i = 0; i < C::NBAR; ++i)
      mbar_init(bar(i), (i >= C::B_DSREADY && i < C::B_DSREADY + NBUF) ? 256u : 1u);
    fence_barrier_init();
    fence_proxy_async_smem();
    if (nt > 0) {
      mbar_arrive_expect_tx(bar(C::B_QDO), 2 * C::Q_BYTES);
      for (int bx = 0; bx < C::NBOX; ++bx) {
        tma_load_4d(smem0 + C::OFF_Q + bx * (BM * 128), &tm_q, bar(C::B_QDO), bx * 64, h,
                    sq.q_row0 + q0, sq.tma_b);
        tma_load_4d(smem0 + C::OFF_DO + bx * (BM * 128), &tm_do, bar(C::B_QDO), bx * 64, h,
                    sq.q_row0 + q0, sq.tma_b);
      }
      load_k(0);
      load_v(0);
    }
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
      for (int n = 1; n < nt; ++n)
        if (!load_k(n) || !load_v(n)) break;
      for (int n = nt - KS < 0 ? 0 : nt - KS; n < nt; ++n)
        if (!mbar_wait(bar(C::B_KFULL + n % KS), (n / KS) & 1)) break;
      for (int n = nt - VS < 0 ? 0 : nt - VS; n < nt; ++n)
        if (!mbar_wait(bar(C::B_VFULL + n % VS), (n / VS) & 1)) break;
      mbar_wait(bar(C::B_QDO), 0);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (nt > 0) {
      constexpr uint32_t idesc_s = idesc_f16(BM, BN, C::FP16, false, false);
      constexpr uint32_t idesc_dq = idesc_f16(BM, D, C::FP16, false, true);
      const uint64_t q_kdesc = sdesc_sw128(smem0 + C::OFF_Q, 16, 1024);
      const uint64_t do_kdesc = sdesc_sw128(smem0 + C::OFF_DO, 16, 1024);
      // S_n = Q K_n^T into the S block of buffer n % NBUF
      auto issue_s = [&](int n) -> bool {
        const int slot = n % KS, bf = n % NBUF;
        const uint64_t k_desc = sdesc_sw128(smem0 + C::OFF_K + slot * C::KV_BYTES, 16, 1024);
        if (!mbar_wait_warp(bar(C::B_KFULL + slot), (n / KS) & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int bx = kk / 4, w = kk % 4;
          mma_ss_warp(tmem + C::TM_S + bf * BN, desc_at(q_kdesc, bx * (BM * 128) + w * 32),
                      desc_at(k_desc, bx * (BN * 128) + w * 32), idesc_s, kk > 0);
        }
        mma_commit_warp(bar(C::B_SFULL + bf));
        return true;
      };
      // dP_n = dO V_n^T into the dP block of buffer n % NBUF
      auto issue_dp = [&](int n) -> bool {
        const int slot = n % VS, bf = n % NBUF;
        const uint64_t v_desc = sdesc_sw128(smem0 + C::OFF_V + slot * C::KV_BYTES, 16, 1024);
        if (!mbar_wait_warp(bar(C::B_VFULL + slot), (n / VS) & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int bx = kk / 4, w = kk % 4;
          mma_ss_warp(tmem + C::TM_DP + bf * BN, desc_at(do_kdesc, bx * (BM * 128) + w * 32),
                      desc_at(v_desc, bx * (BN * 128) + w * 32), idesc_s, kk > 0);
        }
        mma_commit_warp(bar(C::B_DPFULL + bf));
        mma_commit_warp(bar(C::B_VEMPTY + slot));
        return true;
      };
      // dQ += dS_n K_n: dS 16-bit in the first columns of each half of the S
      // block, K_n MN-major (head-dim columns contiguous)
      auto issue_dq = [&](int n) -> bool {
        const int slot = n % KS, bf = n % NBUF, use = n / NBUF;
        const uint64_t k_mn = sdesc_sw128(smem0 + C::OFF_K + slot * C::KV_BYTES, BN * 128, 1024);
        if (!mbar_wait_warp(bar(C::B_DSREADY + bf), use & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const int half = kk / (HW / 16), part = kk % (HW / 16);
          mma_ts_warp(tmem + C::TM_DQ, tmem + C::TM_S + bf * BN + half * HW + part * 8,
                      desc_at(k_mn, kk * 2048), idesc_dq, (n > 0 || kk > 0));
        }
        mma_commit_warp(bar(C::B_KEMPTY + slot));
        return true;
      };
      bool ok = mbar_wait_warp(bar(C::B_QDO), 0) && issue_s(0) && issue_dp(0);
      for (int n = 0; ok && n < nt; ++n) {
        const bool more = n + 1 < nt;
        if (more && !issue_s(n + 1)) { ok = false; break; }
        if (!issue_dq(n)) { ok = false; break; }
        if (more && !issue_dp(n + 1)) { ok = false; break; }
      }
      if (ok) mma_commit_warp(bar(C::B_DONE));
    }
  } else {
    // ------------------------------------------------------------ P, dS
    const int quad = (int)(warp & 3), half = (int)(warp >> 2);
    const int r = quad * 32 + (int)lane;  // query row within the tile == TMEM lane
    const int c0 = half * HW;             // first key column of this warp
    const long long i = (long long)q0 + r;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    // this row's statistics (padding rows: LSE2 = +inf, so P = 0)
    const size_t srow = (size_t)(p.cu_q ? h : b * p.nheads + h) * p.nq_pad + prow0 + q0 + r;
    const float lse2 = p.lse2[srow], dvec = p.dvec[srow];
    const long long vis_lo = i + off - lb;
    const long long vis_hi = min(i + off + rb, (long long)p.seqlen_k - 1);
    const float bk = ALIBI ? -p.alibi[h] * 1.4426950408889634f : 0.f;
    const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
    const uint64_t neg_l2 = f2_pack(-lse2, -lse2);
    const uint64_t neg_d2 = f2_pack(-dvec, -dvec);
    bool ok = true;
    for (int n = 0; n < nt; ++n) {
      const int bf = n % NBUF, use = n / NBUF;
      const long long kc0 = (long long)(lo + n) * BN + c0;  // first key of this warp's columns
      if (!mbar_wait_warp(bar(C::B_SFULL + bf), use & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t s_tmem = tmem + lane_base + C::TM_S + bf * BN + c0;
      float pr[HW];
      {
        uint32_t raw[32];
        tmem_ld32(s_tmem, raw);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < HW; ++c) pr[c] = __uint_as_float(raw[c]);
      }
      const float bd = ALIBI ? (float)(i + off - kc0) : 0.f;
#pragma unroll
      for (int c = 0; c < HW; c += 2) {
        float a0, a1;
        f2_unpack(f2_fma(f2_pack(pr[c], pr[c + 1]), scale2, neg_l2), a0, a1);
        if constexpr (ALIBI) {
          a0 = fmaf(fabsf(bd - (float)c), bk, a0);
          a1 = fmaf(fabsf(bd - (float)(c + 1)), bk, a1);
        }
        pr[c] = ex2(a0);
        pr[c + 1] = ex2(a1);
      }
      if (!(kc0 >= vis_lo && kc0 + HW - 1 <= vis_hi)) {
#pragma unroll
        for (int c = 0; c < HW; ++c)
          if (kc0 + c < vis_lo || kc0 + c > vis_hi) pr[c] = 0.f;
      }
      if (!mbar_wait_warp(bar(C::B_DPFULL + bf), use & 1)) { ok = false; break; }
      tc_fence_after();
      {
        uint32_t raw[32];
        tmem_ld32(tmem + lane_base + C::TM_DP + bf * BN + c0, raw);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < HW; c += 2)
          f2_unpack(f2_mul(f2_pack(pr[c], pr[c + 1]),
                           f2_add(f2_pack(__uint_as_float(raw[c]), __uint_as_float(raw[c + 1])),
                                  neg_d2)),
                    pr[c], pr[c + 1]);
      }
      // dS, 16-bit, over this half's first score columns (already read):
      // the A operand of the dQ product
      uint32_t w[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) w[e] = pack2<C::FP16>(pr[2 * e], pr[2 * e + 1]);
      tmem_st16(s_tmem, w);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(C::B_DSREADY + bf));
    }
    // ------------------------------------------------------------ epilogue
    // This thread's row, head-dim columns [half * 128, half * 128 + 128),
    // added to the fp32 accumulator (dense (batch, seqlen_q, nheads, d),
    // packed (nq_pad, nheads, d) from padded row prow0); bwd_convert applies
    // the scale.  A tile with no visible key adds nothing.
    if (ok && nt > 0) ok = mbar_wait_warp(bar(C::B_DONE), 0);
    if (ok && nt > 0) {
      tc_fence_after();
      const bool row_ok = i < p.seqlen_q;
      float* acc = p.dq_acc +
                   (((size_t)sq.tma_b * pin.seqlen_q + (size_t)(prow0 + i)) * p.nheads + h) * D;
#pragma unroll 1
      for (int c = half * (D / 2); c < (half + 1) * (D / 2); c += 32) {
        uint32_t raw[32];
        tmem_ld32(tmem + lane_base + C::TM_DQ + c, raw);
        tmem_ld_wait();
        if (!row_ok) continue;
        float4* dst = reinterpret_cast<float4*>(acc + c);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float4 a = dst[e];
          a.x += __uint_as_float(raw[4 * e]);
          a.y += __uint_as_float(raw[4 * e + 1]);
          a.z += __uint_as_float(raw[4 * e + 2]);
          a.w += __uint_as_float(raw[4 * e + 3]);
          dst[e] = a;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    // every MMA this warp issued has completed (also on a path that gave
    // up early) before the tensor memory is released
    if (nt > 0) {
      mma_commit_warp(bar(C::B_FLUSH));
      mbar_wait_warp(bar(C::B_FLUSH), 0);
    }
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace attn
