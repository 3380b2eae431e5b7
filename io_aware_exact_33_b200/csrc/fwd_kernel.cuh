// fwd_kernel.cuh - exact attention forward pass for sm_100a.
//
// One CTA computes one 128-row query tile of one (batch, head):
//   O = softmax(Q K^T * scale + mask) V,  LSE = log sum exp(scaled scores)
// streaming the visible K/V tiles through shared memory.  The method is the
// tiled, online-softmax attention described on the pages ("FlashAttention ...
// transformer optimization", items 1-2; FlashAttention-2 page, "Tile-level
// parallelism" and "shared memory"); the mapping onto B200 is this file's:
//
//   warp 4      TMA producer: Q once, then K_j and V_j into rings of
//               shared-memory slots of their own (KSTAGES and VSTAGES
//               deep), each guarded by mbarriers; a K slot is free once S_j
//               has read it, a V slot once O += P_j V_j has, so the next K
//               tiles load while the softmax of this one runs.
//   warp 5      allocates tensor memory; lane 0 issues every tcgen05.mma:
//               S_j = Q K_j^T into one of two TMEM score buffers, and
//               O += P_j V_j with P_j read straight from TMEM.
//   warps 0-3   softmax, one thread per query row (TMEM lane = row): load
//               S_j, mask, running max in log2 units, exp2, running sum,
//               P_j as 16-bit values back into the score buffer; rescale O
//               in TMEM only when the running max grew by more than 8
//               (log2 units), so P stays below 2^8 and the result is the
//               same; at the end O/l, LSE, and a TMA store of O.
//
// Tensor memory (fp32 columns): S0 [0, BN), S1 [BN, 2BN), O [2BN, 2BN + D).
// P_j overwrites the first BN/2 columns of its score buffer as packed
// 16-bit pairs.  MMAs issued by one thread execute in issue order, so S_{j+2}
// (same buffer) is written only after O += P_j V_j has read P_j.
#pragma once

#include <type_traits>

#include "philox.cuh"
#include "sm100.cuh"

namespace attn {

struct FwdParams {
  float* lse;
  int batch, nheads, nheads_kv, seqlen_q, seqlen_k;
  int causal, window_left, window_right;
  float scale_log2;  // softmax_scale * log2(e)
  int num_qblocks;   // work units per (batch, head): query tiles or tile pairs
  int sched_group;   // heads per scheduling group (grouped_lpt)
  // Packed variable-length sequences when cu_q != nullptr (see seq_span):
  // seqlen_q / seqlen_k then hold the longest sequence, total_q / total_k
  // the rows of the packed tensors, lse is (nheads, total_q), and a query
  // tile that ends past its sequence is written through `o` row by row.
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
  uint16_t* o;
  // Per-head positional slopes (nheads floats), or nullptr: scores gain
  // -slope_h * |i + off - j| (kernels instantiated with ALIBI).
  const float* alibi;
  // off = seqlen_k - seqlen_q + pos_offset places the query rows relative to
  // the keys for the masks and the bias (0: bottom-right alignment).
  int pos_offset;
  // Dropout (kernels instantiated with DROP; the contract in philox.cuh):
  // drop_kadd = dropout_kadd(t), drop_scale = 256 / (256 - t).
  unsigned long long drop_seed;
  uint32_t drop_offset, drop_kadd;
  float drop_scale;
};

// Where one softmax thread's dropout bytes come from: generator key and
// offset, head index b * H + h, the thread's query row.
struct DropRow {
  unsigned long long seed;
  uint32_t offset, bh, row, kadd;
};

// Row `row` of query head h of sequence (b, sq) in the LSE output.
__device__ __forceinline__ size_t lse_index(const FwdParams& p, const SeqSpan& sq, int b, int h,
                                            int row) {
  return p.cu_q ? (size_t)h * p.total_q + sq.q_row0 + row
                : ((size_t)b * p.nheads + h) * p.seqlen_q + row;
}



// Range of visible key positions for query rows [q0, q1): keys [jmin, jmax].
struct KeyRange {
  long long jmin, jmax;
};

__device__ __forceinline__ KeyRange visible_keys(int q0, int q1, const FwdParams& p) {
  const long long off = (long long)p.seqlen_k - p.seqlen_q + p.pos_offset;
  const long long kInf = 1ll << 40;
  const long long rb = p.causal ? 0 : (p.window_right >= 0 ? p.window_right : kInf);
  const long long lb = p.window_left >= 0 ? p.window_left : kInf;
  long long jmin = (long long)q0 + off - lb;
  long long jmax = (long long)(q1 - 1) + off + rb;
  if (jmin < 0) jmin = 0;
  if (jmax > (long long)p.seqlen_k - 1) jmax = (long long)p.seqlen_k - 1;
  return {jmin, jmax};
}

template <int D_, int BN_, int KSTAGES_, int VSTAGES_, bool FP16_>
struct FwdCfg {
  static constexpr int D = D_, BN = BN_, KSTAGES = KSTAGES_, VSTAGES = VSTAGES_;
  static constexpr bool FP16 = FP16_;
  static constexpr int BM = 128;
  static constexpr int NBOX = D / 64;              // 64-column (128-byte) boxes per row
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KSTAGES * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + VSTAGES * KV_BYTES;
  // barriers
  static constexpr int B_Q = 0;
  static constexpr int B_KFULL = 1;
  static constexpr int B_VFULL = B_KFULL + KSTAGES;
  static constexpr int B_KEMPTY = B_VFULL + VSTAGES;
  static constexpr int B_VEMPTY = B_KEMPTY + KSTAGES;
  static constexpr int B_SFULL = B_VEMPTY + VSTAGES;  // 2
  static constexpr int B_PREADY = B_SFULL + 2;      // 2
  static constexpr int B_OREADY = B_PREADY + 2;     // 1
  static constexpr int NBAR = B_OREADY + 1;
  static constexpr int OFF_TMEMPTR = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_TMEMPTR + 16 + 1024;  // + alignment slack
  static constexpr int TM_S0 = 0, TM_S1 = BN, TM_O = 2 * BN;
  static constexpr int TMEM_COLS = (2 * BN + D) <= 256 ? 256 : 512;
  static constexpr int THREADS = 192;
  static_assert(D % 64 == 0 && D <= 256, "head dim");
  static_assert(BN % 32 == 0 && BN <= 256, "kv tile");
  static_assert(2 * BN + D <= 512, "tensor memory");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <class C, bool ALIBI>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const FwdParams pin) {
  constexpr int D = C::D, BN = C::BN, BM = C::BM, KS = C::KSTAGES, VS = C::VSTAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem0 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem0 - smem_addr(smem_raw));
  auto bar = [&](int i) -> uint32_t { return smem0 + C::OFF_BAR + 8u * i; };
  volatile uint32_t* tmem_ptr_slot = reinterpret_cast<volatile uint32_t*>(smem_gen + C::OFF_TMEMPTR);

  const uint32_t warp = warp_id(), lane = lane_id();
  // later query tiles see more keys under a causal mask: heaviest first
  const UnitOrder uo = grouped_lpt((int)blockIdx.x, pin.num_qblocks, pin.batch * pin.nheads,
                                   pin.sched_group);
  const int qblock = pin.num_qblocks - 1 - uo.rank;
  const int h = uo.head % pin.nheads, b = uo.head / pin.nheads;
  const SeqSpan sq = seq_span(pin.cu_q, pin.cu_k, pin.total_q, pin.total_k, b, pin.seqlen_q,
                              pin.seqlen_k);
  FwdParams p = pin;  // lengths of this block's sequence
  p.seqlen_q = sq.len_q;
  p.seqlen_k = sq.len_k;
  const int kvh = h / (p.nheads / p.nheads_kv);
  const int q0 = qblock * BM;
  if (q0 >= p.seqlen_q) return;  // past a packed sequence: nothing to do
  const int q1 = min(q0 + BM, p.seqlen_q);
  const bool row_store = p.cu_q != nullptr && q0 + BM > p.seqlen_q;

  const KeyRange kr = visible_keys(q0, q1, p);
  const int t_lo = kr.jmax >= kr.jmin ? (int)(kr.jmin / BN) : 0;
  const int nt = kr.jmax >= kr.jmin ? (int)(kr.jmax / BN) - t_lo + 1 : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NBAR; ++i)
      mbar_init(bar(i), (i == C::B_PREADY || i == C::B_PREADY + 1) ? 128 : 1);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem0 + C::OFF_TMEMPTR, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_o);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nt > 0) {
      mbar_arrive_expect_tx(bar(C::B_Q), C::Q_BYTES);
      for (int bx = 0; bx < C::NBOX; ++bx)
        tma_load_4d(smem0 + C::OFF_Q + bx * (BM * 128), &tm_q, bar(C::B_Q), bx * 64, h,
                    sq.q_row0 + q0, sq.tma_b);
      auto load_k = [&](int t) -> bool {
        const int st = t % KS, n = t / KS;
        if (n > 0 && !mbar_wait(bar(C::B_KEMPTY + st), (n - 1) & 1)) return false;
        mbar_arrive_expect_tx(bar(C::B_KFULL + st), C::KV_BYTES);
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_load_4d(smem0 + C::OFF_K + st * C::KV_BYTES + bx * (BN * 128), &tm_k,
                      bar(C::B_KFULL + st), bx * 64, kvh, sq.k_row0 + (t_lo + t) * BN,
                      sq.tma_b);
        return true;
      };
      auto load_v = [&](int t) -> bool {
        const int st = t % VS, n = t / VS;
        if (n > 0 && !mbar_wait(bar(C::B_VEMPTY + st), (n - 1) & 1)) return false;
        mbar_arrive_expect_tx(bar(C::B_VFULL + st), C::KV_BYTES);
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_load_4d(smem0 + C::OFF_V + st * C::KV_BYTES + bx * (BN * 128), &tm_v,
                      bar(C::B_VFULL + st), bx * 64, kvh, sq.k_row0 + (t_lo + t) * BN,
                      sq.tma_b);
        return true;
      };
      // K runs one tile ahead of V: a V slot still in use (until O += P V
      // of two tiles back) never holds back the next K load.
      bool ok = load_k(0);
      for (int t = 0; ok && t < nt; ++t) {
        if (t + 1 < nt) ok = load_k(t + 1);
        ok = ok && load_v(t);
      }
      // Loads still in flight must land before the CTA can exit: wait (bounded)
      // for the last fill of every slot used.
      for (int t = nt - KS < 0 ? 0 : nt - KS; t < nt; ++t)
        if (!mbar_wait(bar(C::B_KFULL + t % KS), (t / KS) & 1)) break;
      for (int t = nt - VS < 0 ? 0 : nt - VS; t < nt; ++t)
        if (!mbar_wait(bar(C::B_VFULL + t % VS), (t / VS) & 1)) break;
      mbar_wait(bar(C::B_Q), 0);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the issue loop; one elected lane issues.
    if (nt > 0) {
      constexpr uint32_t idesc_qk = idesc_f16(BM, BN, C::FP16, false, false);
      constexpr uint32_t idesc_pv = idesc_f16(BM, D, C::FP16, false, true);
      bool ok = mbar_wait_warp(bar(C::B_Q), 0);
      auto issue_pv = [&](int u) -> bool {
        const int st = u % VS, buf = u & 1;
        if (!mbar_wait_warp(bar(C::B_PREADY + buf), (u >> 1) & 1)) return false;
        if (!mbar_wait_warp(bar(C::B_VFULL + st), (u / VS) & 1)) return false;
        tc_fence_after();
        const uint32_t v_base = smem0 + C::OFF_V + st * C::KV_BYTES;
        const uint32_t p_tmem = tmem + (buf ? C::TM_S1 : C::TM_S0);
        // V tile as the MN-major B operand: 16 key rows (2048 B) per step;
        // 64-column boxes BN*128 bytes apart; 8-row groups 1024 B apart.
        const uint64_t v_desc = sdesc_sw128(v_base, BN * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t bdesc = desc_at(v_desc, kk * 2048);
          mma_ts_warp(tmem + C::TM_O, p_tmem + kk * 8, bdesc, idesc_pv, (u > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit_warp(bar(C::B_OREADY));
        mma_commit_warp(bar(C::B_VEMPTY + st));
        return true;
      };
      for (int t = 0; ok && t < nt; ++t) {
        const int st = t % KS, buf = t & 1;
        if (!mbar_wait_warp(bar(C::B_KFULL + st), (t / KS) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t s_tmem = tmem + (buf ? C::TM_S1 : C::TM_S0);
        const uint64_t q_desc = sdesc_sw128(smem0 + C::OFF_Q, 16, 1024);
        const uint64_t k_desc = sdesc_sw128(smem0 + C::OFF_K + st * C::KV_BYTES, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // K-major operands: 16 columns = 32 bytes per step inside a
          // 128-byte swizzled row; next 64-column box at +rows*128 bytes.
          const int bx = kk / 4, w = kk % 4;
          const uint64_t adesc = desc_at(q_desc, bx * (BM * 128) + w * 32);
          const uint64_t bdesc = desc_at(k_desc, bx * (BN * 128) + w * 32);
          mma_ss_warp(s_tmem, adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit_warp(bar(C::B_SFULL + buf));
        mma_commit_warp(bar(C::B_KEMPTY + st));
        if (t >= 1 && !issue_pv(t - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(nt - 1);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int r = (int)threadIdx.x;  // row within the tile == TMEM lane
    const int i = q0 + r;            // query position
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const long long off = (long long)p.seqlen_k - p.seqlen_q + p.pos_offset;
    const long long kInf = 1ll << 40;
    const long long rb = p.causal ? 0 : (p.window_right >= 0 ? p.window_right : kInf);
    const long long lb = p.window_left >= 0 ? p.window_left : kInf;
    const long long jhi = (long long)i + off + rb;  // visible keys: [jlo, jhi]
    const long long jlo = (long long)i + off - lb;
    const long long blk_hi = (long long)q0 + off + rb;            // every row sees up to here
    const long long blk_lo = (long long)(q0 + BM - 1) + off - lb;  // every row sees from here
    // positional slope in log2 units (negated): bias_c = bk * |bd - c|
    const float bk = ALIBI ? -p.alibi[h] * 1.4426950408889634f : 0.f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < nt; ++t) {
      const int buf = t & 1;
      if (!mbar_wait_warp(bar(C::B_SFULL + buf), (t >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t s_tmem = tmem + lane_base + (buf ? C::TM_S1 : C::TM_S0);
      float s[BN];
#pragma unroll
      for (int c = 0; c < BN; c += 32) {
        uint32_t raw[32];
        tmem_ld32(s_tmem + c, raw);
#pragma unroll
        for (int e = 0; e < 32; ++e) s[c + e] = __uint_as_float(raw[e]);
      }
      tmem_ld_wait();
      const long long k0 = (long long)(t_lo + t) * BN;
      const bool full = (k0 + BN <= p.seqlen_k) && (k0 + BN - 1 <= blk_hi) && (k0 >= blk_lo);
      if (!full) {
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          const long long j = k0 + c;
          if (j >= p.seqlen_k || j > jhi || j < jlo) s[c] = -INFINITY;
        }
      }
      // sl: the factor still to apply to s (the bias case scales up front)
      float sl = p.scale_log2;
      if constexpr (ALIBI) {
        const float bd = (float)((long long)i + off - k0);
#pragma unroll
        for (int c = 0; c < BN; ++c) s[c] = fmaf(s[c], p.scale_log2, bk * fabsf(bd - (float)c));
        sl = 1.f;
      }
      // four independent running maxima (no single dependent chain)
      float mq[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
      for (int c = 4; c < BN; c += 8) {
        mq[0] = max3f(mq[0], s[c], s[c + 1]);
        mq[1] = max3f(mq[1], s[c + 2], s[c + 3]);
        if (c + 4 < BN) {
          mq[2] = max3f(mq[2], s[c + 4], s[c + 5]);
          mq[3] = max3f(mq[3], s[c + 6], s[c + 7]);
        }
      }
      const float mx = max3f(mq[0], mq[1], fmaxf(mq[2], mq[3]));
      const float m_tile = mx * sl;  // scale > 0
      // Keep the old reference max unless the row max grew by more than 8
      // (log2 units); the first tile always sets it.
      float m_use = m, alpha = 1.f;
      if (m_tile > m + 8.f) {
        m_use = m_tile;
        alpha = (m == -INFINITY) ? 0.f : ex2(m - m_tile);
      }
      const float m_sub = (m_use == -INFINITY) ? 0.f : m_use;
      float rs0 = 0.f, rs1 = 0.f;  // two sums: no single dependent chain
      uint32_t packed[BN / 2];
#pragma unroll
      for (int c = 0; c < BN; c += 2) {
        const float p0 = ex2(fmaf(s[c], sl, -m_sub));
        const float p1 = ex2(fmaf(s[c + 1], sl, -m_sub));
        rs0 += p0;
        rs1 += p1;
        packed[c / 2] = pack2<C::FP16>(p0, p1);
      }
      const float rowsum = rs0 + rs1;
      l = l * alpha + rowsum;
      m = m_use;
      // Rescale O (after O += P_{t-1} V_{t-1} has landed) if any row of this
      // warp changed its reference max.
      if (t > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        if (!mbar_wait_warp(bar(C::B_OREADY), (t - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t o_tmem = tmem + lane_base + C::TM_O;
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t raw[32];
          tmem_ld32(o_tmem + c, raw);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * alpha);
          tmem_st32(o_tmem + c, raw);
        }
      }
#pragma unroll
      for (int c = 0; c < BN / 2; c += 16) {
        uint32_t chunk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) chunk[e] = packed[c + e];
        tmem_st16(s_tmem + c, chunk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(C::B_PREADY + buf));
    }
    // ------------------------------------------------------------ epilogue
    if (ok && nt > 0) ok = mbar_wait_warp(bar(C::B_OREADY), (nt - 1) & 1);
    if (ok) {
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const uint32_t o_tmem = tmem + lane_base + C::TM_O;
      const uint32_t row_addr = smem0 + C::OFF_Q + r * 128;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t raw[32];
        if (nt > 0) {
          tmem_ld32(o_tmem + c, raw);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) raw[e] = 0u;
        }
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack2<C::FP16>(__uint_as_float(raw[2 * e]) * inv_l,
                                __uint_as_float(raw[2 * e + 1]) * inv_l);
        if (row_store) {
          if (i < p.seqlen_q)
            store_row32(p.o + ((size_t)(sq.q_row0 + i) * p.nheads + h) * D + c, w);
          continue;
        }
        // 32 columns = 64 bytes = four 16-byte chunks of a 128-byte swizzled row.
        const int bx = c / 64, chunk0 = (c % 64) / 8;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int chunk = (chunk0 + q4) ^ (r & 7);
          st_shared_v4(row_addr + bx * (BM * 128) + chunk * 16, w[4 * q4], w[4 * q4 + 1],
                       w[4 * q4 + 2], w[4 * q4 + 3]);
        }
      }
      fence_proxy_async_smem();
      if (i < p.seqlen_q) {
        const float lse = l > 0.f ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
        p.lse[lse_index(p, sq, b, h, i)] = lse;
      }
    }
    tc_fence_before();
    named_bar_sync(1, 128);
    if (ok && threadIdx.x == 0 && !row_store) {
      for (int bx = 0; bx < C::NBOX; ++bx)
        tma_store_4d(&tm_o, smem0 + C::OFF_Q + bx * (BM * 128), bx * 64, h, sq.q_row0 + q0,
                     sq.tma_b);
      bulk_commit_group();
      bulk_wait_group_read_all();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace attn

namespace attn {

// ---------------------------------------------------------------------------
// Two query tiles per CTA (d <= 128).
//
// Same computation as attn_fwd_kernel, with two 128-row query tiles of one
// (batch, head) sharing each K/V tile, so that the tensor pipe always has
// one tile's MMAs to run while the other tile's softmax warps exponentiate:
//
//   warps 0-3   softmax of query tile 0     warps 4-7   softmax of tile 1
//   warp 8      TMA producer                warp 9      MMA issuer
//
// MMA order per key tile j:  S0_j, PV1_{j-1}, S1_j, PV0_j  (each only where
// tile 0 / tile 1 sees key tile j).  S_i of one key tile is issued after
// PV_i of the previous one, so whenever tile i's softmax runs, its O_i is
// settled in tensor memory and the (conditional) rescale needs no wait.
// Softmax reads its scores twice from tensor memory in 32-column chunks:
// once for the row max, once for exp2 / sum / 16-bit P, which keeps the
// per-thread register footprint small.
//
// Tensor memory: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D).
// ---------------------------------------------------------------------------
template <int D_, int KSTAGES_, int VSTAGES_, bool FP16_>
struct FwdPPCfg {
  static constexpr int D = D_, BN = 128, KSTAGES = KSTAGES_, VSTAGES = VSTAGES_;
  static constexpr bool FP16 = FP16_;
  static constexpr int BM = 128;   // rows per query tile; two tiles per CTA
  static constexpr int NBOX = D / 64;
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_Q = 0;  // two tiles
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + KSTAGES * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + VSTAGES * KV_BYTES;
  static constexpr int B_Q = 0;
  static constexpr int B_KFULL = 1;
  static constexpr int B_VFULL = B_KFULL + KSTAGES;
  static constexpr int B_KEMPTY = B_VFULL + VSTAGES;   // K slot read by its last S MMA
  static constexpr int B_VEMPTY = B_KEMPTY + KSTAGES;  // V slot read by its last PV MMA
  static constexpr int B_SFULL = B_VEMPTY + VSTAGES;   // per query tile
  static constexpr int B_PREADY = B_SFULL + 2;  // per (query tile, half of the key tile), 128 arrivals
  static constexpr int B_OREADY = B_PREADY + 4;  // per query tile
  static constexpr int NBAR = B_OREADY + 2;
  static constexpr int OFF_TMEMPTR = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_TMEMPTR + 16 + 1024;
  static constexpr int TM_S = 0, TM_O = 2 * BN;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 320;
  static_assert(D == 64 || D == 128, "two O tiles must fit tensor memory");
  static_assert(TM_O + 2 * D <= TMEM_COLS, "tensor memory");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// One row's softmax of one key tile, run by each softmax thread (row =
// TMEM lane).  Scores are read from tensor memory 32 columns at a time with
// the next chunk's load in flight.  Pass 1: row max (columns outside
// [vlo, vhi) count as -inf when MASK).  Then the reference max (kept unless
// the row max grew by more than 8 in log2 units) and, if any row of the warp
// moved it, O_i *= alpha in tensor memory.  Pass 2: P = exp2(s*scale*log2e -
// m), the row sum, and 16-bit P written over score columns already read
// (chunk c's P lands in columns [16c, 16c + 16), below the chunk in flight).
// Column pairs of each 32-column chunk whose exponentials go through the
// FMA-pipe polynomial instead of MUFU ex2 (bit i = pair i), on tiles with no
// masked column; the two units then work in parallel.
constexpr uint32_t kPolyPairs = 0x2222u;

// With ALIBI, column c of the tile gains bk * |bd - c| (log2 units): bd is
// the row's position (plus the alignment offset) minus the tile's first key,
// bk the negated slope times log2(e), and `left` says every visible column
// lies left of (or on) the row's diagonal (causal masks).
//  * Row max: when the bias varies by at most 64 across the tile, an upper
//    bound — the raw maximum, scaled, plus the tile's largest bias
//    (bk * distance of bd from [0, BN)); a reference max above the true one
//    only scales P (and l) by a common power of two, so O and LSE are
//    unchanged.  Otherwise the exact maximum of the biased scores.
//  * Exponentials: when, for every row of the warp, all visible columns lie
//    on one side of its diagonal, the bias is linear in the column, b0 +
//    dl * c, and rides in the FMA's addend (one extra packed FMA per column
//    pair); tiles the diagonal crosses add it column by column.
//
// With DROP, P is written to tensor memory with dropped elements zeroed
// (the row sum keeps them: l and the LSE are those of the undropped scores);
// the 1 / (1 - p) factor is applied to O in the epilogue.  The generator's
// integer work then shares the FMA pipe, so no exponential is offloaded to
// the polynomial.
template <bool MASK, bool ALIBI, bool DROP, class C>
__device__ __forceinline__ void softmax_tile(uint32_t s_tmem, uint32_t o_tmem, int n, int vlo,
                                             int vhi, float scale_log2, float m, float& mx,
                                             float& rowsum, float& alpha, float& m_use,
                                             uint32_t pready_half0, uint32_t pready_half1,
                                             float bd, float bk, bool left, const DropRow& dr,
                                             uint32_t k0) {
  constexpr int BN = C::BN, D = C::D;
  auto val = [&](uint32_t bits, int col) -> float {
    return (MASK && (col < vlo || col >= vhi)) ? -INFINITY : __uint_as_float(bits);
  };
  const bool bounded = !ALIBI || (-bk * (float)(BN - 1) <= 64.f);  // uniform: one slope per CTA
  mx = -INFINITY;
  {
    // four independent running maxima, so the 3-input max instructions of
    // a chunk do not form one dependent chain
    float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    uint32_t buf[2][32];
    tmem_ld32(s_tmem, buf[0]);
    tmem_ld_wait();
#pragma unroll
    for (int c = 0; c < BN / 32; ++c) {
      if (c + 1 < BN / 32) tmem_ld32(s_tmem + (c + 1) * 32, buf[(c + 1) & 1]);
      if (bounded) {
#pragma unroll
        for (int e = 0; e < 32; e += 2)
          mq[(e / 2) & 3] = max3f(mq[(e / 2) & 3], val(buf[c & 1][e], c * 32 + e),
                                  val(buf[c & 1][e + 1], c * 32 + e + 1));
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = c * 32 + e;
          mx = fmaxf(mx, fmaf(val(buf[c & 1][e], col), scale_log2, bk * fabsf(bd - (float)col)));
        }
      }
      if (c + 1 < BN / 32) tmem_ld_wait();
    }
    mx = fmaxf(mx, max3f(mq[0], mq[1], fmaxf(mq[2], mq[3])));
  }
  float m_tile = bounded ? mx * scale_log2 : mx;  // scale > 0
  if (ALIBI && bounded) m_tile += bk * fmaxf(fmaxf(-bd, bd - (float)(BN - 1)), 0.f);
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
        f2_unpack(f2_mul(f2_pack(__uint_as_float(raw[e]), __uint_as_float(raw[e + 1])), alpha2), lo, hi);
        raw[e] = __float_as_uint(lo);
        raw[e + 1] = __float_as_uint(hi);
      }
      tmem_st32(o_tmem + c, raw);
    }
    tmem_st_wait();
  }
  // Column pairs go through packed f32x2 FMA / ADD: one instruction computes
  // s*scale*log2e - m for two columns, one adds two P values to two running
  // sums (combined at the end).
  const uint64_t scale2 = f2_pack(scale_log2, scale_log2);
  const uint64_t neg_m2 = f2_pack(-m_sub, -m_sub);
  uint64_t sum2 = f2_pack(0.f, 0.f);
  // linear bias for the whole warp? (b0 = bias at column 0, dl per column)
  bool lin = false;
  uint64_t base2 = neg_m2, step2 = f2_pack(0.f, 0.f);
  if constexpr (ALIBI) {
    const bool right = bd <= 0.f;
    const bool row_left = left || bd >= (float)(BN - 1);
    lin = __all_sync(0xffffffffu, row_left || right);
    const float b0 = row_left ? bk * bd : -bk * bd;
    const float dl = row_left ? -bk : bk;
    base2 = f2_pack(b0 - m_sub, b0 - m_sub);
    step2 = f2_pack(dl, dl);
  }
  auto exp_pass = [&](auto lin_tag) {
    constexpr bool LIN = decltype(lin_tag)::value;
    // linear bias: addend of columns (col, col + 1), advanced by 2 dl a pair
    uint64_t add2 = f2_fma(f2_pack(0.f, 1.f), step2, base2);
    const uint64_t step2x2 = f2_add(step2, step2);
    uint32_t buf[2][32];
    tmem_ld32(s_tmem, buf[0]);
    tmem_ld_wait();
#pragma unroll
    for (int c = 0; c < BN / 32; ++c) {
      // this row's random bytes for the chunk's 32 columns (DROP), made
      // before the next chunk's load is in flight
      [[maybe_unused]] uint32_t kw[8];
      if constexpr (DROP) {
        uint32_t a[4], z[4];
        dropout_row16(dr.seed, dr.offset, dr.bh, dr.row, k0 + 32u * c, a);
        dropout_row16(dr.seed, dr.offset, dr.bh, dr.row, k0 + 32u * c + 16u, z);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          kw[k] = a[k];
          kw[4 + k] = z[k];
        }
      }
      if (c + 1 < BN / 32) tmem_ld32(s_tmem + (c + 1) * 32, buf[(c + 1) & 1]);
      uint32_t w[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const int col = c * 32 + e;
        const uint64_t x2 = f2_pack(val(buf[c & 1][e], col), val(buf[c & 1][e + 1], col + 1));
        float a0, a1, p0, p1;
        if constexpr (LIN) {
          f2_unpack(f2_fma(x2, scale2, add2), a0, a1);
          add2 = f2_add(add2, step2x2);
        } else {
          f2_unpack(f2_fma(x2, scale2, neg_m2), a0, a1);
          if constexpr (ALIBI) {
            a0 = fmaf(fabsf(bd - (float)col), bk, a0);
            a1 = fmaf(fabsf(bd - (float)(col + 1)), bk, a1);
          }
        }
        if (!MASK && !DROP && ((kPolyPairs >> (e / 2)) & 1)) {
          exp2_poly2(a0, a1, p0, p1);
        } else {
          p0 = ex2(a0);
          p1 = ex2(a1);
        }
        sum2 = f2_add(sum2, f2_pack(p0, p1));
        w[e / 2] = pack2<C::FP16>(p0, p1);
        if constexpr (DROP)
          w[e / 2] &= dropout_pair_mask(dropout_keep_bits(kw[e / 4], (e / 2) & 1, dr.kadd));
      }
      if (c + 1 < BN / 32) tmem_ld_wait();
      tmem_st16(s_tmem + c * 16, w);
      if (c == BN / 64 - 1 || c == BN / 32 - 1) {
        // this half of P is in tensor memory: let its PV MMAs start
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(c == BN / 32 - 1 ? pready_half1 : pready_half0);
      }
    }
  };
  if (ALIBI && lin)
    exp_pass(std::true_type{});
  else
    exp_pass(std::false_type{});
  {
    float s0, s1;
    f2_unpack(sum2, s0, s1);
    rowsum = s0 + s1;
  }
}

template <class C, bool ALIBI, bool DROP>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_fwd_pp_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                       const FwdParams pin) {
  constexpr int D = C::D, BN = C::BN, BM = C::BM, KS = C::KSTAGES, VS = C::VSTAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem0 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem0 - smem_addr(smem_raw));
  auto bar = [&](int i) -> uint32_t { return smem0 + C::OFF_BAR + 8u * i; };
  volatile uint32_t* tmem_ptr_slot = reinterpret_cast<volatile uint32_t*>(smem_gen + C::OFF_TMEMPTR);

  const uint32_t warp = warp_id(), lane = lane_id();
  // later query tiles see more keys under a causal mask: heaviest first
  const UnitOrder uo = grouped_lpt((int)blockIdx.x, pin.num_qblocks, pin.batch * pin.nheads,
                                   pin.sched_group);
  const int pair = pin.num_qblocks - 1 - uo.rank;
  const int h = uo.head % pin.nheads, b = uo.head / pin.nheads;
  const SeqSpan sq = seq_span(pin.cu_q, pin.cu_k, pin.total_q, pin.total_k, b, pin.seqlen_q,
                              pin.seqlen_k);
  FwdParams p = pin;  // lengths of this block's sequence
  p.seqlen_q = sq.len_q;
  p.seqlen_k = sq.len_k;
  if (2 * pair * BM >= p.seqlen_q) return;  // past a packed sequence: nothing to do
  const int kvh = h / (p.nheads / p.nheads_kv);

  // Key-tile range [lo_i, hi_i) of each query tile; union [ulo, uhi).
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

  // K and V slots are released separately: K_j after key tile j's last S
  // MMA (same iteration), V_j after its last PV MMA (up to one later).  K
  // runs one tile ahead of V in the issue order, so a V slot that is still
  // in use never holds back the next K load.
  auto load_k = [&](int t) -> bool {
    const int st = t % KS, n = t / KS;
    if (n > 0 && !mbar_wait(bar(C::B_KEMPTY + st), (n - 1) & 1)) return false;
    mbar_arrive_expect_tx(bar(C::B_KFULL + st), C::KV_BYTES);
    for (int bx = 0; bx < C::NBOX; ++bx)
      tma_load_4d(smem0 + C::OFF_K + st * C::KV_BYTES + bx * (BN * 128), &tm_k,
                  bar(C::B_KFULL + st), bx * 64, kvh, sq.k_row0 + (ulo + t) * BN, sq.tma_b);
    return true;
  };
  auto load_v = [&](int t) -> bool {
    const int st = t % VS, n = t / VS;
    if (n > 0 && !mbar_wait(bar(C::B_VEMPTY + st), (n - 1) & 1)) return false;
    mbar_arrive_expect_tx(bar(C::B_VFULL + st), C::KV_BYTES);
    for (int bx = 0; bx < C::NBOX; ++bx)
      tma_load_4d(smem0 + C::OFF_V + st * C::KV_BYTES + bx * (BN * 128), &tm_v,
                  bar(C::B_VFULL + st), bx * 64, kvh, sq.k_row0 + (ulo + t) * BN, sq.tma_b);
    return true;
  };

  // The producer lane initialises the barriers and starts the Q and first K
  // loads before the block-wide barrier, so that their latency overlaps the
  // tensor-memory allocation and the barrier itself.
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
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_load_4d(smem0 + C::OFF_Q + i * C::Q_BYTES + bx * (BM * 128), &tm_q, bar(C::B_Q),
                      bx * 64, h, sq.q_row0 + qs[i], sq.tma_b);
      load_k(0);  // first use of its slot: no wait
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
      bool go = true;  // Q and K_0 are on their way
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
    // The whole warp runs the issue loop (its values stay warp-uniform); one
    // elected lane issues each MMA and commit.
    if (nt > 0) {
      constexpr uint32_t idesc_qk = idesc_f16(BM, BN, C::FP16, false, false);
      constexpr uint32_t idesc_pv = idesc_f16(BM, D, C::FP16, false, true);
      int ns[2] = {0, 0};  // S MMAs issued per query tile
      int np[2] = {0, 0};  // PV MMAs issued per query tile
      auto in = [&](int i, int j) { return j >= lo[i] && j < hi[i]; };
      auto issue_s = [&](int i, int j, bool last_use) {
        const int st = (j - ulo) % KS;
        const uint64_t q_desc = sdesc_sw128(smem0 + C::OFF_Q + i * C::Q_BYTES, 16, 1024);
        const uint64_t k_desc = sdesc_sw128(smem0 + C::OFF_K + st * C::KV_BYTES, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int bx = kk / 4, w = kk % 4;
          mma_ss_warp(tmem + C::TM_S + i * BN, desc_at(q_desc, bx * (BM * 128) + w * 32),
                 desc_at(k_desc, bx * (BN * 128) + w * 32), idesc_qk, kk > 0);
        }
        mma_commit_warp(bar(C::B_SFULL + i));
        if (last_use) mma_commit_warp(bar(C::B_KEMPTY + st));
        ++ns[i];
      };
      // O_i += P_i V_j in two halves of the key tile, each issued as soon as
      // the softmax warps have stored that half of P.
      auto issue_pv = [&](int i, int j, bool last_use) -> bool {
        const int u = j - ulo, st = u % VS;
        if (!mbar_wait_warp(bar(C::B_VFULL + st), (u / VS) & 1)) return false;
        const uint64_t v_desc = sdesc_sw128(smem0 + C::OFF_V + st * C::KV_BYTES, BN * 128, 1024);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          if (!mbar_wait_warp(bar(C::B_PREADY + 2 * i + hf), np[i] & 1)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = hf * (BN / 32); kk < (hf + 1) * (BN / 32); ++kk)
            mma_ts_warp(tmem + C::TM_O + i * D, tmem + C::TM_S + i * BN + kk * 8,
                   desc_at(v_desc, kk * 2048), idesc_pv,
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
    const int r = quad * 32 + (int)lane;  // row within the tile == TMEM lane
    const int row = q_i + r;             // query position
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t s_tmem = tmem + lane_base + C::TM_S + i * BN;
    const uint32_t o_tmem = tmem + lane_base + C::TM_O + i * D;
    const long long off = (long long)p.seqlen_k - p.seqlen_q + p.pos_offset;
    const long long kInf = 1ll << 40;
    const long long rb = p.causal ? 0 : (p.window_right >= 0 ? p.window_right : kInf);
    const long long lb = p.window_left >= 0 ? p.window_left : kInf;
    const long long jhi = (long long)row + off + rb;  // visible keys: [jlo, jhi]
    const long long jlo = (long long)row + off - lb;
    const long long blk_hi = (long long)q_i + off + rb;
    const long long blk_lo = (long long)(q_i + BM - 1) + off - lb;
    const int n_i = hi_i - lo_i;
    // positional slope in log2 units (negated): bias of column c = bk * |bd - c|
    const float bk = ALIBI ? -p.alibi[h] * 1.4426950408889634f : 0.f;
    // seed, offset and kadd straight from the kernel parameters (constant
    // bank), so they hold no registers across the key loop
    const DropRow dr{pin.drop_seed, pin.drop_offset, (uint32_t)(b * pin.nheads + h),
                     (uint32_t)row, pin.drop_kadd};
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int n = 0; n < n_i; ++n) {
      if (!mbar_wait_warp(bar(C::B_SFULL + i), n & 1)) { ok = false; break; }
      tc_fence_after();
      const long long k0 = (long long)(lo_i + n) * BN;
      const bool full = (k0 + BN <= p.seqlen_k) && (k0 + BN - 1 <= blk_hi) && (k0 >= blk_lo);
      // Visible columns of this row within the key tile: [vlo, vhi).
      int vlo = 0, vhi = BN;
      if (!full) {
        const long long a = jlo - k0, z = min(jhi, (long long)p.seqlen_k - 1) - k0 + 1;
        vlo = (int)max(0ll, min((long long)BN, a));
        vhi = (int)max(0ll, min((long long)BN, z));
      }
      float mx, rowsum, alpha, m_use;
      const uint32_t ph0 = bar(C::B_PREADY + 2 * i), ph1 = bar(C::B_PREADY + 2 * i + 1);
      const float bd = ALIBI ? (float)((long long)row + off - k0) : 0.f;
      if (full)
        softmax_tile<false, ALIBI, DROP, C>(s_tmem, o_tmem, n, vlo, vhi, p.scale_log2, m, mx,
                                            rowsum, alpha, m_use, ph0, ph1, bd, bk, p.causal != 0,
                                            dr, (uint32_t)k0);
      else
        softmax_tile<true, ALIBI, DROP, C>(s_tmem, o_tmem, n, vlo, vhi, p.scale_log2, m, mx,
                                           rowsum, alpha, m_use, ph0, ph1, bd, bk, p.causal != 0,
                                           dr, (uint32_t)k0);
      l = l * alpha + rowsum;
      m = m_use;
    }
    // ------------------------------------------------------------ epilogue
    if (ok && n_i > 0) ok = mbar_wait_warp(bar(C::B_OREADY + i), (n_i - 1) & 1);
    // A tile with no visible key still had its Q loaded (when the CTA has
    // work): that load must land before the staging area is overwritten.
    if (ok && n_i == 0 && nt > 0) ok = mbar_wait_warp(bar(C::B_Q), 0);
    const uint32_t stage = smem0 + C::OFF_Q + i * C::Q_BYTES;  // Q_i is no longer read
    const bool row_store = p.cu_q != nullptr && q_i + BM > p.seqlen_q;
    if (ok) {
      tc_fence_after();
      const float inv_l = l > 0.f ? (DROP ? p.drop_scale : 1.f) / l : 0.f;
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
          w[e] = pack2<C::FP16>(__uint_as_float(raw[2 * e]) * inv_l,
                                __uint_as_float(raw[2 * e + 1]) * inv_l);
        if (row_store) {
          if (row < p.seqlen_q)
            store_row32(p.o + ((size_t)(sq.q_row0 + row) * p.nheads + h) * D + c, w);
          continue;
        }
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
        p.lse[lse_index(p, sq, b, h, row)] = lse;
      }
    }
    tc_fence_before();
    named_bar_sync(1 + i, 128);
    if (ok && quad == 0 && lane == 0 && q_i < p.seqlen_q && !row_store) {
      for (int bx = 0; bx < C::NBOX; ++bx)
        tma_store_4d(&tm_o, stage + bx * (BM * 128), bx * 64, h, sq.q_row0 + q_i, sq.tma_b);
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
