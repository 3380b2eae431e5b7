// fwd_fp8_kernel.cuh - exact attention forward with E4M3 (FP8) inputs.
//
// FlashAttention-3's FP8 forward is named on the FlashAttention four-
// generations page (hardware and dtype section).  Q, K and V arrive as E4M3
// codes with one float scale per tensor (x ~ scale * e4m3(code)); the result
// is attention over those dequantized values, written as bf16 or fp16:
//     S = (q8 k8^T) * (q_scale * k_scale * softmax_scale),
//     O = softmax(S) (v_scale * v8),  LSE as the 16-bit forward's.
//
// The same two-query-tile pipeline as attn_fwd_pp_kernel (fwd_kernel.cuh),
// with the 8-bit differences:
//   * TMA boxes of 128 E4M3 columns (one 128-byte swizzled row per head-dim
//     row, d = 128); half the shared memory per tile of the 16-bit kernel.
//   * S = Q K^T by tcgen05.mma kind::f8f6f4 (E4M3 x E4M3 -> f32, both
//     operands K-major), four K = 32 steps of 32 bytes.
//   * P is rounded to E4M3 (satfinite; P <= 2^8 under the conditional
//     rescale, inside E4M3's range of 448) and stored four per tensor-memory
//     column (byte k = key 4c + k): 32 columns for a 128-key tile.
//   * O += P V with P from tensor memory and V as an MN-major E4M3 operand
//     (keys x d with d contiguous, as loaded), K = 32 keys per step.
//   * v_scale is applied with 1/l in the epilogue.
// Dense batches only (no packed sequences), no positional slopes, no
// dropout; headdim 128.
#pragma once

#include "fwd_kernel.cuh"

namespace attn {

// D[tmem] (+)= A * B, E4M3 operands; warp-wide issue as mma_ss_warp.
__device__ __forceinline__ void mma_f8_ss_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_f8_ts_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of kind::f8f6f4 with E4M3 A and B and an f32
// accumulator (format code 0 = E4M3 in both operand fields).
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4)                                  // D = f32
         | (0u << 7) | (0u << 10)                   // A, B = E4M3
         | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16)
         | (static_cast<uint32_t>(N >> 3) << 17)   // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);  // M / 16
}

// Four floats to four E4M3 bytes, `a` in the lowest byte; round to nearest
// even, saturating at +-448.
__device__ __forceinline__ uint32_t pack4_e4m3(float a, float b, float c, float d) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(r)
      : "f"(a), "f"(b), "f"(c), "f"(d));
  return r;
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

template <int KSTAGES_, int VSTAGES_, bool FP16_OUT_>
struct FwdF8Cfg {
  static constexpr int D = 128, BN = 128, BM = 128, KSTAGES = KSTAGES_, VSTAGES = VSTAGES_;
  static constexpr bool FP16 = FP16_OUT_;  // output dtype
  static constexpr int Q_BYTES = BM * D;   // one byte per element, 128-byte rows
  static constexpr int KV_BYTES = BN * D;
  static constexpr int O_BYTES = BM * D * 2;  // 16-bit output staging (two 64-column boxes)
  static constexpr int OFF_Q = 0;             // two query tiles
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + KSTAGES * KV_BYTES;
  static constexpr int OFF_O = OFF_V + VSTAGES * KV_BYTES;  // two output staging tiles
  static constexpr int OFF_BAR = OFF_O + 2 * O_BYTES;
  static constexpr int B_Q = 0;
  static constexpr int B_KFULL = 1;
  static constexpr int B_VFULL = B_KFULL + KSTAGES;
  static constexpr int B_KEMPTY = B_VFULL + VSTAGES;
  static constexpr int B_VEMPTY = B_KEMPTY + KSTAGES;
  static constexpr int B_SFULL = B_VEMPTY + VSTAGES;
  static constexpr int B_PREADY = B_SFULL + 2;
  static constexpr int B_OREADY = B_PREADY + 4;
  static constexpr int NBAR = B_OREADY + 2;
  static constexpr int OFF_TMEMPTR = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_TMEMPTR + 16 + 1024;
  static constexpr int TM_S = 0, TM_O = 2 * BN;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 320;
  static_assert(TM_O + 2 * D <= TMEM_COLS, "tensor memory");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// One row's softmax of one key tile (as softmax_tile in fwd_kernel.cuh,
// without slopes): row max, conditional rescale of O, then P = exp2(s *
// scale - m) rounded to E4M3 and stored four per column (chunk c of 32 keys
// in columns [8c, 8c + 8)), signalling each half of the tile.
template <bool MASK, class C>
__device__ __forceinline__ void softmax_tile_e4m3(uint32_t s_tmem, uint32_t o_tmem, int n, int vlo,
                                                  int vhi, float scale_log2, float m, float& rowsum,
                                                  float& alpha, float& m_use,
                                                  uint32_t pready_half0, uint32_t pready_half1) {
  constexpr int BN = C::BN, D = C::D;
  auto val = [&](uint32_t bits, int col) -> float {
    return (MASK && (col < vlo || col >= vhi)) ? -INFINITY : __uint_as_float(bits);
  };
  float mx = -INFINITY;
  {
    // four independent running maxima (no single dependent chain)
    float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    uint32_t buf[2][32];
    tmem_ld32(s_tmem, buf[0]);
    tmem_ld_wait();
#pragma unroll
    for (int c = 0; c < BN / 32; ++c) {
      if (c + 1 < BN / 32) tmem_ld32(s_tmem + (c + 1) * 32, buf[(c + 1) & 1]);
#pragma unroll
      for (int e = 0; e < 32; e += 2)
        mq[(e / 2) & 3] = max3f(mq[(e / 2) & 3], val(buf[c & 1][e], c * 32 + e),
                                val(buf[c & 1][e + 1], c * 32 + e + 1));
      if (c + 1 < BN / 32) tmem_ld_wait();
    }
    mx = max3f(mq[0], mq[1], fmaxf(mq[2], mq[3]));
  }
  const float m_tile = mx * scale_log2;  // scale > 0
  m_use = m;
  alpha = 1.f;
  if (m_tile > m + 8.f) {
    m_use = m_tile;
    alpha = (m == -INFINITY) ? 0.f : ex2(m - m_tile);
  }
  const float m_sub = (m_use == -INFINITY) ? 0.f : m_use;
  if (n > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
    for (int c = 0; c < D; c += 32) {
      uint32_t raw[32];
      tmem_ld32(o_tmem + c, raw);
      tmem_ld_wait();
      const uint64_t alpha2 = f2_pack(alpha, alpha);
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        float lo, hi;
        f2_unpack(f2_mul(f2_pack(__uint_as_float(raw[e]), __uint_as_float(raw[e + 1])), alpha2),
                  lo, hi);
        raw[e] = __float_as_uint(lo);
        raw[e + 1] = __float_as_uint(hi);
      }
      tmem_st32(o_tmem + c, raw);
    }
    tmem_st_wait();
  }
  const uint64_t scale2 = f2_pack(scale_log2, scale_log2);
  const uint64_t neg_m2 = f2_pack(-m_sub, -m_sub);
  uint64_t sum2 = f2_pack(0.f, 0.f);
  uint32_t buf[2][32];
  tmem_ld32(s_tmem, buf[0]);
  tmem_ld_wait();
#pragma unroll
  for (int c = 0; c < BN / 32; ++c) {
    if (c + 1 < BN / 32) tmem_ld32(s_tmem + (c + 1) * 32, buf[(c + 1) & 1]);
    float pv[32];
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const int col = c * 32 + e;
      float a0, a1;
      f2_unpack(f2_fma(f2_pack(val(buf[c & 1][e], col), val(buf[c & 1][e + 1], col + 1)), scale2,
                       neg_m2),
                a0, a1);
      if (!MASK && ((kPolyPairs >> (e / 2)) & 1)) {
        exp2_poly2(a0, a1, pv[e], pv[e + 1]);
      } else {
        pv[e] = ex2(a0);
        pv[e + 1] = ex2(a1);
      }
      sum2 = f2_add(sum2, f2_pack(pv[e], pv[e + 1]));
    }
    uint32_t w[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) w[q] = pack4_e4m3(pv[4 * q], pv[4 * q + 1], pv[4 * q + 2], pv[4 * q + 3]);
    if (c + 1 < BN / 32) tmem_ld_wait();
    tmem_st8(s_tmem + c * 8, w);
    if (c == BN / 64 - 1 || c == BN / 32 - 1) {
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(c == BN / 32 - 1 ? pready_half1 : pready_half0);
    }
  }
  float s0, s1;
  f2_unpack(sum2, s0, s1);
  rowsum = s0 + s1;
}

// FwdParams as for the 16-bit kernels (scale_log2 already includes the Q
// and K scales); v_scale multiplies O.
template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_fwd_e4m3_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                         const FwdParams p, const float v_scale) {
  constexpr int D = C::D, BN = C::BN, BM = C::BM, KS = C::KSTAGES, VS = C::VSTAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem0 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem0 - smem_addr(smem_raw));
  auto bar = [&](int i) -> uint32_t { return smem0 + C::OFF_BAR + 8u * i; };
  volatile uint32_t* tmem_ptr_slot = reinterpret_cast<volatile uint32_t*>(smem_gen + C::OFF_TMEMPTR);

  const uint32_t warp = warp_id(), lane = lane_id();
  const UnitOrder uo = grouped_lpt((int)blockIdx.x, p.num_qblocks, p.batch * p.nheads,
                                   p.sched_group);
  const int pair = p.num_qblocks - 1 - uo.rank;
  const int h = uo.head % p.nheads, b = uo.head / p.nheads;
  const int kvh = h / (p.nheads / p.nheads_kv);

  int lo[2], hi[2], qs[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    qs[i] = (2 * pair + i) * BM;
    const int q1 = min(qs[i] + BM, p.seqlen_q);
    lo[i] = hi[i] = 0;
    if (qs[i] < q1) {
      const KeyRange kr = visible_keys(qs[i], q1, p);
      if (kr.jmax >= kr.jmin) {
        lo[i] = (int)(kr.jmin / BN);
        hi[i] = (int)(kr.jmax / BN) + 1;
      }
    }
  }
  const bool has0 = hi[0] > lo[0], has1 = hi[1] > lo[1];
  const int ulo = has0 && has1 ? min(lo[0], lo[1]) : (has0 ? lo[0] : lo[1]);
  const int uhi = has0 && has1 ? max(hi[0], hi[1]) : (has0 ? hi[0] : hi[1]);
  const int nt = (has0 || has1) ? uhi - ulo : 0;

  auto load_k = [&](int t) -> bool {
    const int st = t % KS, n = t / KS;
    if (n > 0 && !mbar_wait(bar(C::B_KEMPTY + st), (n - 1) & 1)) return false;
    mbar_arrive_expect_tx(bar(C::B_KFULL + st), C::KV_BYTES);
    tma_load_4d(smem0 + C::OFF_K + st * C::KV_BYTES, &tm_k, bar(C::B_KFULL + st), 0, kvh,
                (ulo + t) * BN, b);
    return true;
  };
  auto load_v = [&](int t) -> bool {
    const int st = t % VS, n = t / VS;
    if (n > 0 && !mbar_wait(bar(C::B_VEMPTY + st), (n - 1) & 1)) return false;
    mbar_arrive_expect_tx(bar(C::B_VFULL + st), C::KV_BYTES);
    tma_load_4d(smem0 + C::OFF_V + st * C::KV_BYTES, &tm_v, bar(C::B_VFULL + st), 0, kvh,
                (ulo + t) * BN, b);
    return true;
  };

  if (warp == 8 && lane == 0) {
    for (int i = 0; i < C::NBAR; ++i)
      mbar_init(bar(i), (i >= C::B_PREADY && i < C::B_PREADY + 4) ? 128 : 1);
    fence_barrier_init();
    fence_proxy_async_smem();
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_o);
    if (nt > 0) {
      mbar_arrive_expect_tx(bar(C::B_Q), 2 * C::Q_BYTES);
      for (int i = 0; i < 2; ++i)
        tma_load_4d(smem0 + C::OFF_Q + i * C::Q_BYTES, &tm_q, bar(C::B_Q), 0, h, qs[i], b);
      load_k(0);
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
      bool go = true;
      for (int t = 0; go && t < nt; ++t) {
        if (t + 1 < nt) go = load_k(t + 1);
        go = go && load_v(t);
      }
      for (int t = nt - KS < 0 ? 0 : nt - KS; t < nt; ++t)
        if (!mbar_wait(bar(C::B_KFULL + t % KS), (t / KS) & 1)) break;
      for (int t = nt - VS < 0 ? 0 : nt - VS; t < nt; ++t)
        if (!mbar_wait(bar(C::B_VFULL + t % VS), (t / VS) & 1)) break;
      mbar_wait(bar(C::B_Q), 0);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (nt > 0) {
      constexpr uint32_t idesc_qk = idesc_e4m3(BM, BN, false, false);
      constexpr uint32_t idesc_pv = idesc_e4m3(BM, D, false, true);
      int np[2] = {0, 0};
      auto in = [&](int i, int j) { return j >= lo[i] && j < hi[i]; };
      auto issue_s = [&](int i, int j, bool last_use) {
        const int st = (j - ulo) % KS;
        const uint64_t q_desc = sdesc_sw128(smem0 + C::OFF_Q + i * C::Q_BYTES, 16, 1024);
        const uint64_t k_desc = sdesc_sw128(smem0 + C::OFF_K + st * C::KV_BYTES, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)  // 32 bytes of each 128-byte row per step
          mma_f8_ss_warp(tmem + C::TM_S + i * BN, desc_at(q_desc, kk * 32),
                         desc_at(k_desc, kk * 32), idesc_qk, kk > 0);
        mma_commit_warp(bar(C::B_SFULL + i));
        if (last_use) mma_commit_warp(bar(C::B_KEMPTY + st));
      };
      auto issue_pv = [&](int i, int j, bool last_use) -> bool {
        const int u = j - ulo, st = u % VS;
        if (!mbar_wait_warp(bar(C::B_VFULL + st), (u / VS) & 1)) return false;
        const uint64_t v_desc = sdesc_sw128(smem0 + C::OFF_V + st * C::KV_BYTES, BN * 128, 1024);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          if (!mbar_wait_warp(bar(C::B_PREADY + 2 * i + hf), np[i] & 1)) return false;
          tc_fence_after();
          // 32 keys per step: 8 tensor-memory columns of P, 32 V rows
#pragma unroll
          for (int kk = hf * (BN / 64); kk < (hf + 1) * (BN / 64); ++kk)
            mma_f8_ts_warp(tmem + C::TM_O + i * D, tmem + C::TM_S + i * BN + kk * 8,
                           desc_at(v_desc, kk * 32 * 128), idesc_pv,
                           (np[i] > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit_warp(bar(C::B_OREADY + i));
        if (last_use) mma_commit_warp(bar(C::B_VEMPTY + st));
        ++np[i];
        return true;
      };
      bool ok = mbar_wait_warp(bar(C::B_Q), 0);
      for (int j = ulo; ok && j < uhi; ++j) {
        const int u = j - ulo, st = u % KS;
        if (!mbar_wait_warp(bar(C::B_KFULL + st), (u / KS) & 1)) { ok = false; break; }
        tc_fence_after();
        if (in(0, j)) issue_s(0, j, !in(1, j));
        if (j > ulo && in(1, j - 1) && !issue_pv(1, j - 1, true)) { ok = false; break; }
        if (in(1, j)) issue_s(1, j, true);
        if (in(0, j) && !issue_pv(0, j, !in(1, j))) { ok = false; break; }
      }
      if (ok && in(1, uhi - 1)) issue_pv(1, uhi - 1, true);
    }
  } else {
    // ------------------------------------------------------------ softmax (tile i)
    const int i = (int)(warp >> 2);
    const int quad = (int)(warp & 3);
    const int q_i = i ? qs[1] : qs[0], lo_i = i ? lo[1] : lo[0], hi_i = i ? hi[1] : hi[0];
    const int r = quad * 32 + (int)lane;
    const int row = q_i + r;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t s_tmem = tmem + lane_base + C::TM_S + i * BN;
    const uint32_t o_tmem = tmem + lane_base + C::TM_O + i * D;
    const long long off = (long long)p.seqlen_k - p.seqlen_q + p.pos_offset;
    const long long kInf = 1ll << 40;
    const long long rb = p.causal ? 0 : (p.window_right >= 0 ? p.window_right : kInf);
    const long long lb = p.window_left >= 0 ? p.window_left : kInf;
    const long long jhi = (long long)row + off + rb;
    const long long jlo = (long long)row + off - lb;
    const long long blk_hi = (long long)q_i + off + rb;
    const long long blk_lo = (long long)(q_i + BM - 1) + off - lb;
    const int n_i = hi_i - lo_i;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int n = 0; n < n_i; ++n) {
      if (!mbar_wait_warp(bar(C::B_SFULL + i), n & 1)) { ok = false; break; }
      tc_fence_after();
      const long long k0 = (long long)(lo_i + n) * BN;
      const bool full = (k0 + BN <= p.seqlen_k) && (k0 + BN - 1 <= blk_hi) && (k0 >= blk_lo);
      int vlo = 0, vhi = BN;
      if (!full) {
        const long long a = jlo - k0, z = min(jhi, (long long)p.seqlen_k - 1) - k0 + 1;
        vlo = (int)max(0ll, min((long long)BN, a));
        vhi = (int)max(0ll, min((long long)BN, z));
      }
      float rowsum, alpha, m_use;
      const uint32_t ph0 = bar(C::B_PREADY + 2 * i), ph1 = bar(C::B_PREADY + 2 * i + 1);
      if (full)
        softmax_tile_e4m3<false, C>(s_tmem, o_tmem, n, vlo, vhi, p.scale_log2, m, rowsum, alpha,
                                    m_use, ph0, ph1);
      else
        softmax_tile_e4m3<true, C>(s_tmem, o_tmem, n, vlo, vhi, p.scale_log2, m, rowsum, alpha,
                                   m_use, ph0, ph1);
      l = l * alpha + rowsum;
      m = m_use;
    }
    // ------------------------------------------------------------ epilogue
    if (ok && n_i > 0) ok = mbar_wait_warp(bar(C::B_OREADY + i), (n_i - 1) & 1);
    const uint32_t stage = smem0 + C::OFF_O + i * C::O_BYTES;
    if (ok) {
      tc_fence_after();
      const float mul = l > 0.f ? v_scale / l : 0.f;
      const uint32_t row_addr = stage + r * 128;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t raw[32];
        if (n_i > 0) {
          tmem_ld32(o_tmem + c, raw);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) raw[e] = 0u;
        }
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack2<C::FP16>(__uint_as_float(raw[2 * e]) * mul,
                                __uint_as_float(raw[2 * e + 1]) * mul);
        const int bx = c / 64, chunk0 = (c % 64) / 8;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int chunk = (chunk0 + q4) ^ (r & 7);
          st_shared_v4(row_addr + bx * (BM * 128) + chunk * 16, w[4 * q4], w[4 * q4 + 1],
                       w[4 * q4 + 2], w[4 * q4 + 3]);
        }
      }
      fence_proxy_async_smem();
      if (row < p.seqlen_q) {
        const float lse = l > 0.f ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
        p.lse[((size_t)b * p.nheads + h) * p.seqlen_q + row] = lse;
      }
    }
    tc_fence_before();
    named_bar_sync(1 + i, 128);
    if (ok && quad == 0 && lane == 0 && q_i < p.seqlen_q) {
      for (int bx = 0; bx < 2; ++bx)
        tma_store_4d(&tm_o, stage + bx * (BM * 128), bx * 64, h, q_i, b);
      bulk_commit_group();
      bulk_wait_group_read_all();
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
