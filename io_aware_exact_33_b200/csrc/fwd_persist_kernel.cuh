// fwd_persist_kernel.cuh - persistent forward kernel for head dims 64 and
// 128, for workloads whose work units are short (sliding windows, packed
// sequences of a few thousand tokens), where the fixed cost of a one-shot
// block (setup, the first Q / K loads, the pipeline's fill and drain, the
// epilogue) weighs against its few key tiles.
//
// Same computation as the two-tile forward (two 128-row query tiles of one
// (batch, head) share every K/V tile; two softmax warpgroups alternate with
// the tensor pipe), but the grid is one CTA per SM and each CTA takes work
// units (query-tile pairs) one after another: CTA c takes units c, c + G,
// c + 2G, ... (G = grid size) of the grouped longest-first order, so the
// heaviest units are spread over all SMs first (load balance without a
// counter, and every role of the CTA computes the same sequence).  Across
// unit boundaries:
//
//   * the producer loads the next unit's Q tiles and first K/V tiles while
//     the current unit is still computing (each Q slot is released by the
//     MMA warp after its last S MMA of the unit);
//   * the MMA warp issues one continuous stream over (unit, key tile)
//     iterations, S0_j, PV1_{j-1}, S1_j, PV0_j, across unit boundaries, so
//     warpgroup 0 starts the next unit while warpgroup 1 finishes the last
//     key tile of the current one;
//   * O is stored straight from registers to global memory, row by row, so
//     the epilogue needs no shared memory and no barrier across warps; each
//     warpgroup releases its O accumulator (O_FREE) as soon as it has read
//     it, and the next unit's first PV MMA of that tile waits for that.
//
//   warps 0-3   softmax + epilogue of tile 0    warps 4-7   tile 1
//   warp 8      TMA producer                    warp 9      MMA issuer
//
// Barrier phase bookkeeping: every ring position (K, V, Q_i, S_i, PV_i,
// O_FREE_i) counts its uses over the CTA's lifetime, and each side waits
// for each phase in order, never more than one phase behind.  Q_i, QEMPTY_i
// and O_FREE_i count only units in which tile i has work.  No positional
// slopes, no dropout (the dispatcher uses the one-shot kernel for those).
#pragma once
#include "fwd_kernel.cuh"
#include "sm100.cuh"

namespace attn {

template <int D_, int KSTAGES_, int VSTAGES_, bool FP16_>
struct FwdPersistCfg {
  static constexpr int D = D_, BN = 128, KSTAGES = KSTAGES_, VSTAGES = VSTAGES_;
  static constexpr bool FP16 = FP16_;
  static constexpr int BM = 128;  // rows per query tile; two tiles per unit
  static constexpr int NBOX = D / 64;
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_Q = 0;  // two tiles
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + KSTAGES * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + VSTAGES * KV_BYTES;
  static constexpr int B_QFULL = 0;                      // per tile
  static constexpr int B_QEMPTY = B_QFULL + 2;           // per tile: last S MMA of a unit
  static constexpr int B_KFULL = B_QEMPTY + 2;
  static constexpr int B_KEMPTY = B_KFULL + KSTAGES;
  static constexpr int B_VFULL = B_KEMPTY + KSTAGES;
  static constexpr int B_VEMPTY = B_VFULL + VSTAGES;
  static constexpr int B_SFULL = B_VEMPTY + VSTAGES;     // per tile
  static constexpr int B_PREADY = B_SFULL + 2;           // per (tile, half), 128 arrivals
  static constexpr int B_OREADY = B_PREADY + 4;          // per tile
  static constexpr int B_OFREE = B_OREADY + 2;           // per tile, 128 arrivals
  static constexpr int NBAR = B_OFREE + 2;
  static constexpr int OFF_TMEMPTR = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_TMEMPTR + 16 + 1024;
  static constexpr int TM_S = 0, TM_O = 2 * BN;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 320;
  static_assert(D == 64 || D == 128, "two O tiles must fit tensor memory");
  static_assert(TM_O + 2 * D <= TMEM_COLS, "tensor memory");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Geometry of work unit L (a pair of query tiles of one (batch, head)).
struct FwdUnit {
  SeqSpan sq;           // this unit's sequence (its lengths are sq.len_q / len_k)
  int b, h, kvh;
  int qs[2], lo[2], hi[2];  // first query row, key-tile range [lo, hi) per tile
  int ulo, uhi, nt;     // union of the key-tile ranges, its length
  bool live;            // the unit has query rows
};

template <class C>
__device__ __forceinline__ FwdUnit fwd_unit(int L, const FwdParams& pin) {
  constexpr int BM = C::BM, BN = C::BN;
  FwdUnit u;
  // later query tiles see more keys under a causal mask: heaviest first
  const UnitOrder uo = grouped_lpt(L, pin.num_qblocks, pin.batch * pin.nheads, pin.sched_group);
  const int pair = pin.num_qblocks - 1 - uo.rank;
  u.h = uo.head % pin.nheads;
  u.b = uo.head / pin.nheads;
  u.kvh = u.h / (pin.nheads / pin.nheads_kv);
  u.sq = seq_span(pin.cu_q, pin.cu_k, pin.total_q, pin.total_k, u.b, pin.seqlen_q, pin.seqlen_k);
  u.live = 2 * pair * BM < u.sq.len_q;
  FwdParams ps = pin;  // this sequence's lengths, for visible_keys
  ps.seqlen_q = u.sq.len_q;
  ps.seqlen_k = u.sq.len_k;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    u.qs[i] = (2 * pair + i) * BM;
    const int q1 = min(u.qs[i] + BM, u.sq.len_q);
    u.lo[i] = u.hi[i] = 0;
    if (u.qs[i] < q1) {
      const KeyRange kr = visible_keys(u.qs[i], q1, ps);
      if (kr.jmax >= kr.jmin) {
        u.lo[i] = (int)(kr.jmin / BN);
        u.hi[i] = (int)(kr.jmax / BN) + 1;
      }
    }
  }
  const bool has0 = u.hi[0] > u.lo[0], has1 = u.hi[1] > u.lo[1];
  u.ulo = has0 && has1 ? min(u.lo[0], u.lo[1]) : (has0 ? u.lo[0] : u.lo[1]);
  u.uhi = has0 && has1 ? max(u.hi[0], u.hi[1]) : (has0 ? u.hi[0] : u.hi[1]);
  u.nt = (u.live && (has0 || has1)) ? u.uhi - u.ulo : 0;
  return u;
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_fwd_persist_kernel(const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const FwdParams pin,
                            int total_units) {
  constexpr int D = C::D, BN = C::BN, BM = C::BM, KS = C::KSTAGES, VS = C::VSTAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem0 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem0 - smem_addr(smem_raw));
  auto bar = [&](int i) -> uint32_t { return smem0 + C::OFF_BAR + 8u * i; };
  volatile uint32_t* tmem_ptr_slot = reinterpret_cast<volatile uint32_t*>(smem_gen + C::OFF_TMEMPTR);
  const uint32_t warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NBAR; ++i) {
      uint32_t count = 1;
      if (i >= C::B_PREADY && i < C::B_PREADY + 4) count = 128;
      if (i >= C::B_OFREE && i < C::B_OFREE + 2) count = 128;
      mbar_init(bar(i), count);
    }
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem0 + C::OFF_TMEMPTR, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr_slot;

  // This CTA's units: blockIdx.x, then every gridDim.x-th one after it, in
  // the grouped longest-first order (every role walks the same sequence).
  const int stride = (int)gridDim.x;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int kt = 0, vt = 0;    // K / V tiles loaded so far
      int qn[2] = {0, 0};    // Q_i loads so far
      bool ok = true;
      for (int L = (int)blockIdx.x; ok && L < total_units; L += stride) {
        const FwdUnit u = fwd_unit<C>(L, pin);
        if (u.nt == 0) continue;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          if (!ok || u.hi[i] <= u.lo[i]) continue;
          if (qn[i] > 0 && !mbar_wait(bar(C::B_QEMPTY + i), (qn[i] - 1) & 1)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(C::B_QFULL + i), C::Q_BYTES);
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_4d(smem0 + C::OFF_Q + i * C::Q_BYTES + bx * (BM * 128), &tm_q,
                        bar(C::B_QFULL + i), bx * 64, u.h, u.sq.q_row0 + u.qs[i], u.sq.tma_b);
          ++qn[i];
        }
        // K runs one tile ahead of V: a V slot still in use never holds back
        // the next K load.
        auto load_k = [&](int t) -> bool {
          const int pos = kt + t, st = pos % KS, n = pos / KS;
          if (n > 0 && !mbar_wait(bar(C::B_KEMPTY + st), (n - 1) & 1)) return false;
          mbar_arrive_expect_tx(bar(C::B_KFULL + st), C::KV_BYTES);
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_4d(smem0 + C::OFF_K + st * C::KV_BYTES + bx * (BN * 128), &tm_k,
                        bar(C::B_KFULL + st), bx * 64, u.kvh, u.sq.k_row0 + (u.ulo + t) * BN,
                        u.sq.tma_b);
          return true;
        };
        auto load_v = [&](int t) -> bool {
          const int pos = vt + t, st = pos % VS, n = pos / VS;
          if (n > 0 && !mbar_wait(bar(C::B_VEMPTY + st), (n - 1) & 1)) return false;
          mbar_arrive_expect_tx(bar(C::B_VFULL + st), C::KV_BYTES);
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_4d(smem0 + C::OFF_V + st * C::KV_BYTES + bx * (BN * 128), &tm_v,
                        bar(C::B_VFULL + st), bx * 64, u.kvh, u.sq.k_row0 + (u.ulo + t) * BN,
                        u.sq.tma_b);
          return true;
        };
        ok = ok && load_k(0);
        for (int t = 0; ok && t < u.nt; ++t) {
          if (t + 1 < u.nt) ok = load_k(t + 1);
          ok = ok && load_v(t);
        }
        kt += u.nt;
        vt += u.nt;
      }
      // Loads still in flight must land before the CTA exits.
      for (int pos = kt - KS < 0 ? 0 : kt - KS; pos < kt; ++pos)
        if (!mbar_wait(bar(C::B_KFULL + pos % KS), (pos / KS) & 1)) break;
      for (int pos = vt - VS < 0 ? 0 : vt - VS; pos < vt; ++pos)
        if (!mbar_wait(bar(C::B_VFULL + pos % VS), (pos / VS) & 1)) break;
      for (int i = 0; i < 2; ++i)
        if (qn[i] > 0) mbar_wait(bar(C::B_QFULL + i), (qn[i] - 1) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the issue loop (its values stay warp-uniform); one
    // elected lane issues each MMA and commit.
    constexpr uint32_t idesc_qk = idesc_f16(BM, BN, C::FP16, false, false);
    constexpr uint32_t idesc_pv = idesc_f16(BM, D, C::FP16, false, true);
    int kpos = 0, vpos = 0;   // K / V tiles consumed
    int qn[2] = {0, 0};       // units with work for tile i (Q_i phases)
    int pc[2] = {0, 0};       // PV_i issued (PREADY_i phases)
    int pvu[2] = {0, 0};      // units whose PV_i began (O_FREE_i phases)
    // PV1 of the previous iteration, issued after the next S0.
    bool pend = false;
    int pend_v = 0;
    bool pend_first = false;
    bool ok = true;
    auto issue_s = [&](int i, int kslot, bool last_use) {
      const uint64_t q_desc = sdesc_sw128(smem0 + C::OFF_Q + i * C::Q_BYTES, 16, 1024);
      const uint64_t k_desc = sdesc_sw128(smem0 + C::OFF_K + kslot * C::KV_BYTES, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int bx = kk / 4, w = kk % 4;
        mma_ss_warp(tmem + C::TM_S + i * BN, desc_at(q_desc, bx * (BM * 128) + w * 32),
                    desc_at(k_desc, bx * (BN * 128) + w * 32), idesc_qk, kk > 0);
      }
      mma_commit_warp(bar(C::B_SFULL + i));
      if (last_use) mma_commit_warp(bar(C::B_KEMPTY + kslot));
    };
    // O_i (+)= P_i V in two halves of the key tile, each issued as soon as
    // the softmax warps have stored that half of P.  The first PV_i of a
    // unit overwrites O_i: it waits until the previous unit's epilogue of
    // tile i has read O_i out.
    auto issue_pv = [&](int i, int v, bool first, bool last_use) -> bool {
      const int st = v % VS;
      if (first) {
        if (pvu[i] > 0 && !mbar_wait_warp(bar(C::B_OFREE + i), (pvu[i] - 1) & 1)) return false;
        ++pvu[i];
      }
      if (!mbar_wait_warp(bar(C::B_VFULL + st), (v / VS) & 1)) return false;
      const uint64_t v_desc = sdesc_sw128(smem0 + C::OFF_V + st * C::KV_BYTES, BN * 128, 1024);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        if (!mbar_wait_warp(bar(C::B_PREADY + 2 * i + hf), pc[i] & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = hf * (BN / 32); kk < (hf + 1) * (BN / 32); ++kk)
          mma_ts_warp(tmem + C::TM_O + i * D, tmem + C::TM_S + i * BN + kk * 8,
                      desc_at(v_desc, kk * 2048), idesc_pv, (!first || kk > 0) ? 1u : 0u);
      }
      mma_commit_warp(bar(C::B_OREADY + i));
      if (last_use) mma_commit_warp(bar(C::B_VEMPTY + st));
      ++pc[i];
      return true;
    };
    for (int L = (int)blockIdx.x; ok && L < total_units; L += stride) {
      const FwdUnit u = fwd_unit<C>(L, pin);
      if (u.nt == 0) {
        // An empty unit: issue the deferred PV1 now rather than with the
        // next unit that has work (warpgroup 1 is waiting for it).
        if (pend && !issue_pv(1, pend_v, pend_first, true)) { ok = false; break; }
        pend = false;
        continue;
      }
      auto in = [&](int i, int jj) { return jj >= u.lo[i] && jj < u.hi[i]; };
      bool first_s[2] = {true, true}, first_pv[2] = {true, true};
      for (int jj = u.ulo; ok && jj < u.uhi; ++jj) {
        const int kslot = kpos % KS;
        if (!mbar_wait_warp(bar(C::B_KFULL + kslot), (kpos / KS) & 1)) { ok = false; break; }
        tc_fence_after();
        const bool a0 = in(0, jj), a1 = in(1, jj);
        if (a0) {
          if (first_s[0]) {
            if (!mbar_wait_warp(bar(C::B_QFULL + 0), qn[0] & 1)) { ok = false; break; }
            tc_fence_after();
            first_s[0] = false;
          }
          issue_s(0, kslot, !a1);
          if (jj + 1 == u.hi[0]) mma_commit_warp(bar(C::B_QEMPTY + 0));
        }
        if (pend && !issue_pv(1, pend_v, pend_first, true)) { ok = false; break; }
        pend = false;
        if (a1) {
          if (first_s[1]) {
            if (!mbar_wait_warp(bar(C::B_QFULL + 1), qn[1] & 1)) { ok = false; break; }
            tc_fence_after();
            first_s[1] = false;
          }
          issue_s(1, kslot, true);
          if (jj + 1 == u.hi[1]) mma_commit_warp(bar(C::B_QEMPTY + 1));
        }
        if (a0 && !issue_pv(0, vpos, first_pv[0], !a1)) { ok = false; break; }
        if (a0) first_pv[0] = false;
        if (a1) {
          pend = true;
          pend_v = vpos;
          pend_first = first_pv[1];
          first_pv[1] = false;
        }
        if (!a0 && !a1) {  // not reached (the two tiles' key ranges leave no gap)
          mma_commit_warp(bar(C::B_KEMPTY + kslot));
          mma_commit_warp(bar(C::B_VEMPTY + vpos % VS));
        }
        ++kpos;
        ++vpos;
      }
#pragma unroll
      for (int i = 0; i < 2; ++i)
        if (u.hi[i] > u.lo[i]) ++qn[i];
    }
    if (ok && pend) issue_pv(1, pend_v, pend_first, true);
  } else {
    // ------------------------------------------------------------ softmax + epilogue (tile i)
    const int i = (int)(warp >> 2);
    const int quad = (int)(warp & 3);
    const int r = quad * 32 + (int)lane;  // row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t s_tmem = tmem + lane_base + C::TM_S + i * BN;
    const uint32_t o_tmem = tmem + lane_base + C::TM_O + i * D;
    const uint32_t ph0 = bar(C::B_PREADY + 2 * i), ph1 = bar(C::B_PREADY + 2 * i + 1);
    int sn = 0;  // S_i tiles consumed (SFULL_i / OREADY_i phases)
    bool ok = true;
    for (int L = (int)blockIdx.x; ok && L < total_units; L += stride) {
      const FwdUnit u = fwd_unit<C>(L, pin);
      const int len_q = u.sq.len_q, len_k = u.sq.len_k;
      // (selects, not indexing: keeps the unit in registers)
      const int q_i = i ? u.qs[1] : u.qs[0];
      const int lo_i = i ? u.lo[1] : u.lo[0];
      const int n_i = (i ? u.hi[1] : u.hi[0]) - lo_i;
      if (!u.live || q_i >= len_q) continue;  // no rows of this tile
      const int row = q_i + r;  // query position
      const long long off = (long long)len_k - len_q + pin.pos_offset;
      const long long kInf = 1ll << 40;
      const long long rb = pin.causal ? 0 : (pin.window_right >= 0 ? pin.window_right : kInf);
      const long long lb = pin.window_left >= 0 ? pin.window_left : kInf;
      const long long jhi = (long long)row + off + rb;  // visible keys: [jlo, jhi]
      const long long jlo = (long long)row + off - lb;
      const long long blk_hi = (long long)q_i + off + rb;
      const long long blk_lo = (long long)(q_i + BM - 1) + off - lb;
      float m = -INFINITY, l = 0.f;
      for (int n = 0; n < n_i; ++n) {
        if (!mbar_wait_warp(bar(C::B_SFULL + i), sn & 1)) { ok = false; break; }
        ++sn;
        tc_fence_after();
        const long long k0 = (long long)(lo_i + n) * BN;
        const bool full = (k0 + BN <= len_k) && (k0 + BN - 1 <= blk_hi) && (k0 >= blk_lo);
        // Visible columns of this row within the key tile: [vlo, vhi).
        int vlo = 0, vhi = BN;
        if (!full) {
          const long long a = jlo - k0, z = min(jhi, (long long)len_k - 1) - k0 + 1;
          vlo = (int)max(0ll, min((long long)BN, a));
          vhi = (int)max(0ll, min((long long)BN, z));
        }
        float mx, rowsum, alpha, m_use;
        const DropRow dr{0ull, 0u, 0u, 0u, 0u};  // no dropout here
        if (full)
          softmax_tile<false, false, false, C>(s_tmem, o_tmem, n, vlo, vhi, pin.scale_log2, m,
                                               mx, rowsum, alpha, m_use, ph0, ph1, 0.f, 0.f,
                                               pin.causal != 0, dr, (uint32_t)k0);
        else
          softmax_tile<true, false, false, C>(s_tmem, o_tmem, n, vlo, vhi, pin.scale_log2, m,
                                              mx, rowsum, alpha, m_use, ph0, ph1, 0.f, 0.f,
                                              pin.causal != 0, dr, (uint32_t)k0);
        l = l * alpha + rowsum;
        m = m_use;
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      // O / l from tensor memory to registers, O_i released, then stored row
      // by row (rows past the sequence are not written).
      if (n_i > 0 && !mbar_wait_warp(bar(C::B_OREADY + i), (sn - 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      // token row of this query: packed rows from the sequence start, dense
      // rows from the batch entry's start
      const size_t tok = pin.cu_q ? (size_t)u.sq.q_row0 + row : (size_t)u.b * len_q + row;
      uint16_t* dst = pin.o + (tok * pin.nheads + u.h) * D;
      const bool in_seq = row < len_q;
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
        if (n_i > 0 && c + 32 == D) {
          tc_fence_before();
          mbar_arrive(bar(C::B_OFREE + i));
        }
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack2<C::FP16>(__uint_as_float(raw[2 * e]) * inv_l,
                                __uint_as_float(raw[2 * e + 1]) * inv_l);
        if (in_seq) store_row32(dst + c, w);
      }
      if (in_seq) {
        const float lse = l > 0.f ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
        const size_t li = pin.cu_q ? (size_t)u.h * pin.total_q + tok
                                   : ((size_t)u.b * pin.nheads + u.h) * len_q + row;
        pin.lse[li] = lse;
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
