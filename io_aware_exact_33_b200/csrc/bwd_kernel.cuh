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
// Main kernel roles (448 threads):
//   warp 8      TMA producer: K_j, V_j once; Q_i (with its LSE2 statistics)
//               and dO_i (with Dvec) per query tile through rings of their own.
//   warp 9      TMEM allocation; issues the five MMAs per tile (one elected
//               lane): S^T = K Q^T, dP^T = V dO^T, dV += P^T dO, dK += dS^T Q,
//               and dQ^T = K^T dS^T (d = 128) or dQ = dS K (d = 64).  With two
//               buffers it issues tile t+1's S^T before tile t's gradient
//               MMAs and its dP^T after them, so the tensor pipe works on one
//               tile while the compute warps exponentiate the other.
//   warps 0-7   two warps per tensor-memory lane quadrant (one thread per key
//               row), each owning half of the tile's query columns:
//               P^T = exp2(S^T*scale*log2e - LSE2) back into tensor memory as
//               the 16-bit A operand of dV; dS = P o (dP - Dvec) into tensor
//               memory beside it (the A operand of dK) and into shared
//               memory (an MN-major operand of dQ); finally dK, dV out
//               through TMA.
//   warps 10-13 dQ drain: each tile's dQ block (which reuses that tile's dP
//               block) out of tensor memory into the fp32 accumulator with
//               TMA reduce-adds (other key tiles add to the same rows), off
//               the compute warps' path.
#pragma once

#include <cuda_fp16.h>

#include "philox.cuh"
#include "sm100.cuh"

namespace attn {

struct BwdWorkspace {
  size_t dvec_off, lse2_off, lsb_off, dvb_off, dq_off, total;
  long long nq_pad;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Per-query statistics of one padded query row in the form the main kernel's
// MMAs take them (bf16 kernels without dropout): 16 bf16 values, the first
// three a split v = hi + mid + lo of the value that the extra K = 16 step of
// the S^T (v = -LSE2 / (scale log2 e)) or dP^T (v = -Dvec) product adds to
// every key row; the rest zero.
constexpr int kSlabCols = 16;
constexpr int kSlabRowBytes = kSlabCols * 2;

// The arrays after the fp32 Dvec / LSE2 rows (rows = statistics rows, each
// nq_pad long): the two bf16 slabs, then the fp32 dQ accumulator.
__host__ __device__ inline void bwd_workspace_tail(BwdWorkspace& w, size_t stat_rows,
                                                   size_t acc_elems) {
  const size_t rows4 = stat_rows * (size_t)w.nq_pad * 4;
  w.dvec_off = 0;
  w.lse2_off = align_up(rows4, 256);
  w.lsb_off = w.lse2_off + align_up(rows4, 256);
  w.dvb_off = w.lsb_off + align_up(stat_rows * (size_t)w.nq_pad * kSlabRowBytes, 256);
  w.dq_off = w.dvb_off + align_up(stat_rows * (size_t)w.nq_pad * kSlabRowBytes, 256);
  w.total = w.dq_off + align_up(acc_elems * 4, 256);
}

// Workspace: Dvec and LSE2 as (batch*nheads, nq_pad) fp32 with nq_pad a
// multiple of 128 (TMA-aligned rows), their bf16 slabs (batch*nheads,
// nq_pad, 16), then the fp32 dQ accumulator (batch, seqlen_q, nheads,
// headdim).  Packed sequences: see bwd_workspace_layout_packed.
__host__ __device__ inline BwdWorkspace bwd_workspace_layout(int batch, int nheads, int seqlen_q,
                                                            int headdim) {
  BwdWorkspace w;
  w.nq_pad = ((long long)seqlen_q + 127) / 128 * 128;
  bwd_workspace_tail(w, (size_t)batch * nheads, (size_t)batch * seqlen_q * nheads * headdim);
  return w;
}

// Packed sequences: sequence b's rows start at padded row
// packed_row0(cu_q[b], b) = align4(cu_q[b]) + 136 b, a multiple of 4 (TMA
// alignment of the fp32 rows) with >= 128 rows of slack after every sequence,
// so a query tile that ends past its sequence reads and adds only slack rows.
// Dvec and LSE2 are (nheads, nq_pad), the slabs (nheads, nq_pad, 16) and the
// dQ accumulator is (nq_pad, nheads, headdim), nq_pad = packed_rows(total_q,
// batch).
__host__ __device__ inline long long packed_row0(int cu_b, int b) {
  return (((long long)cu_b + 3) & ~3ll) + 136ll * b;
}
__host__ __device__ inline long long packed_rows(int total_q, int batch) {
  return (((long long)total_q + 3) & ~3ll) + 136ll * batch + 128;
}
__host__ __device__ inline BwdWorkspace bwd_workspace_layout_packed(int total_q, int batch,
                                                                   int nheads, int headdim) {
  BwdWorkspace w;
  w.nq_pad = packed_rows(total_q, batch);
  bwd_workspace_tail(w, (size_t)nheads, (size_t)w.nq_pad * nheads * headdim);
  return w;
}

struct BwdParams {
  const float* lse;
  float* dvec;
  float* lse2;
  // bf16 slabs of -LSE2 / scale_log2 and -Dvec (kSlabCols per padded row),
  // written instead of dvec / lse2 when `fold` is set (bf16, no dropout).
  uint16_t* lse_slab;
  uint16_t* dvec_slab;
  int fold;
  float* dq_acc;
  int batch, nheads, nheads_kv, seqlen_q, seqlen_k, headdim;
  int causal, window_left, window_right;
  float scale_log2;
  float softmax_scale;
  long long nq_pad;
  int num_kblocks;   // key tiles per (batch, kv head): the work units
  int num_qblocks;   // 128-row query tiles per (batch, head): the units of the d = 256 dQ kernel
  int sched_group;   // kv heads per scheduling group (grouped_lpt)
  // Packed variable-length sequences when cu_q != nullptr (see seq_span and
  // packed_row0): seqlen_q / seqlen_k then hold the longest sequence,
  // total_q / total_k the rows of the packed tensors, lse is (nheads,
  // total_q), and a key tile that ends past its sequence writes dk / dv row
  // by row.
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
  uint16_t* dk;
  uint16_t* dv;
  // When set, tm_dk / tm_dv map float32 (batch, seqlen_k, nheads_kv, headdim)
  // buffers and the epilogue adds dK (x scale) and dV into them (TMA
  // reduce-add) instead of storing them in the input dtype; dense only.
  int acc_f32;
  // Per-head positional slopes (nheads floats), or nullptr: scores gain
  // -slope_h * |i + off - j| (kernel instantiated with ALIBI).
  const float* alibi;
  // off = seqlen_k - seqlen_q + pos_offset places the query rows relative to
  // the keys for the masks and the bias (0: bottom-right alignment).
  int pos_offset;
  // Dropout (kernel instantiated with DROP; the contract in philox.cuh):
  // drop_kadd = dropout_kadd(t), drop_scale = 256 / (256 - t).
  unsigned long long drop_seed;
  uint32_t drop_offset, drop_kadd;
  float drop_scale;
};

// Packed layout: the sequence owning padded row `pr` (the last b with
// packed_row0 <= pr) and the sequence owning token row `t` (the last b with
// cu_q[b] <= t), by binary search over the clamped offsets.
__device__ inline int packed_seq_of_row(const BwdParams& p, long long pr) {
  int lo = 0, hi = p.batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    const int c = min(max(__ldg(p.cu_q + mid), 0), p.total_q);
    if (packed_row0(c, mid) <= pr) lo = mid; else hi = mid - 1;
  }
  return lo;
}
__device__ inline int packed_seq_of_token(const BwdParams& p, long long t) {
  int lo = 0, hi = p.batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    const int c = min(max(__ldg(p.cu_q + mid), 0), p.total_q);
    if (c <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ------------------------------------------------------------ preprocess
// fp32 dot product of eight 16-bit values of `a` and `b` (16 bytes each).
template <bool FP16>
__device__ __forceinline__ float dot8(uint4 a, uint4 b) {
  const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
  float acc = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float a0, a1, b0, b1;
    if constexpr (FP16) {
      a0 = __half2float(__ushort_as_half((unsigned short)(av[k] & 0xFFFFu)));
      a1 = __half2float(__ushort_as_half((unsigned short)(av[k] >> 16)));
      b0 = __half2float(__ushort_as_half((unsigned short)(bv[k] & 0xFFFFu)));
      b1 = __half2float(__ushort_as_half((unsigned short)(bv[k] >> 16)));
    } else {
      a0 = __uint_as_float(av[k] << 16);
      a1 = __uint_as_float(av[k] & 0xFFFF0000u);
      b0 = __uint_as_float(bv[k] << 16);
      b1 = __uint_as_float(bv[k] & 0xFFFF0000u);
    }
    acc = fmaf(a0, b0, acc);
    acc = fmaf(a1, b1, acc);
  }
  return acc;
}

// bf16 bits of x, round to nearest even.
__device__ __forceinline__ uint32_t bf16_bits(float x) { return pack2<false>(x, 0.f) & 0xFFFFu; }

// One slab row: x split into three bf16 values hi + mid + lo (each the
// bf16 rounding of what the previous ones leave; the differences are exact
// in fp32, so the sum carries 24 significant bits), then 13 zeros.
__device__ __forceinline__ void write_slab_row(uint16_t* dst, float x) {
  const uint32_t hi = bf16_bits(x);
  const float r1 = x - __uint_as_float(hi << 16);
  const uint32_t mid = bf16_bits(r1);
  const float r2 = r1 - __uint_as_float(mid << 16);
  const uint32_t lo = bf16_bits(r2);
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = make_uint4(hi | (mid << 16), lo, 0u, 0u);
  d[1] = make_uint4(0u, 0u, 0u, 0u);
}

// Rows of the padded (b, h, i) range, headdim / 8 lanes per row with one
// 16-byte load of O and of dO each: Dvec_i = sum_c dO_ic O_ic and
// LSE2_i = LSE_i * log2(e); padding rows get 0 and +inf (P = 0 there).  With
// p.fold the same values go to the bf16 slabs instead (write_slab_row).  All
// threads then zero the dQ accumulator.
template <bool FP16>
__global__ void __launch_bounds__(256) bwd_preprocess(const uint16_t* __restrict__ o,
                                                      const uint16_t* __restrict__ dout,
                                                      BwdParams p, long long n_rows,
                                                      long long n_zero4) {
  const int lpr = p.headdim / 8;          // lanes per row: 8 (d = 64) or 16 (d = 128)
  const int rpw = 32 / lpr;               // rows per warp step
  const int lane = threadIdx.x & 31;
  const int sub = lane % lpr;
  const long long warp_global = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long row0 = warp_global * rpw; row0 < n_rows; row0 += nwarps * rpw) {
    const long long row = row0 + lane / lpr;
    const bool in_range = row < n_rows;
    const long long ip = row % p.nq_pad;
    const long long bh = row / p.nq_pad;
    int h = 0, b = 0;
    long long i = 0, tok = 0;  // row within the sequence; row of the o / dout / lse tensors
    bool valid = false;
    if (in_range) {
      if (p.cu_q) {
        h = (int)bh;
        b = packed_seq_of_row(p, ip);
        const SeqSpan sq = seq_span(p.cu_q, p.cu_k, p.total_q, p.total_k, b, 0, 0);
        i = ip - packed_row0(sq.q_row0, b);
        valid = i >= 0 && i < sq.len_q;
        tok = sq.q_row0 + i;
      } else {
        h = (int)(bh % p.nheads);
        b = (int)(bh / p.nheads);
        i = ip;
        valid = i < p.seqlen_q;
        tok = (long long)b * p.seqlen_q + i;
      }
    }
    float acc = 0.f;
    if (valid) {
      const size_t base = ((size_t)tok * p.nheads + h) * p.headdim + sub * 8;
      acc = dot8<FP16>(*reinterpret_cast<const uint4*>(o + base),
                       *reinterpret_cast<const uint4*>(dout + base));
    }
    for (int s = lpr / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (in_range && sub == 0) {
      float l2 = INFINITY;
      if (valid) {
        const float l = p.cu_q ? p.lse[(size_t)h * p.total_q + tok]
                               : p.lse[((size_t)b * p.nheads + h) * p.seqlen_q + i];
        l2 = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
      }
      if (p.fold) {
        // Rows with no visible key or past the sequence get 0: the main
        // kernel masks every one of their elements.
        const float x = (valid && l2 != INFINITY) ? -l2 / p.scale_log2 : 0.f;
        write_slab_row(p.lse_slab + (size_t)row * kSlabCols, x);
        write_slab_row(p.dvec_slab + (size_t)row * kSlabCols, valid ? -acc : 0.f);
      } else {
        p.dvec[row] = valid ? acc : 0.f;
        p.lse2[row] = l2;
      }
    }
  }
  float4* z = reinterpret_cast<float4*>(p.dq_acc);
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  for (long long k = tid; k < n_zero4; k += nthreads) z[k] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ------------------------------------------------------------ convert
// dQ = scale * accumulator, four elements per step.  Packed sequences: token
// row t of sequence b reads padded row packed_row0(cu_q[b], b) + t - cu_q[b].
template <bool FP16>
__global__ void __launch_bounds__(256) bwd_convert(const float* __restrict__ acc,
                                                   uint16_t* __restrict__ dq, long long n4,
                                                   float scale, BwdParams p) {
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  const long long row_len = (long long)p.nheads * p.headdim;
  for (long long k = tid; k < n4; k += nthreads) {
    long long src = k;
    if (p.cu_q) {
      const long long e = 4 * k, t = e / row_len;
      const int b = packed_seq_of_token(p, t);
      const long long c = min(max(__ldg(p.cu_q + b), 0), p.total_q);
      src = ((packed_row0((int)c, b) + (t - c)) * row_len + e % row_len) / 4;
    }
    const float4 a = reinterpret_cast<const float4*>(acc)[src];
    uint2 w;
    w.x = pack2<FP16>(a.x * scale, a.y * scale);
    w.y = pack2<FP16>(a.z * scale, a.w * scale);
    reinterpret_cast<uint2*>(dq)[k] = w;
  }
}

// ------------------------------------------------------------ main kernel
// Tile sizes: BN = 128 key rows per CTA (the tensor-memory lane count);
// BM query rows per step.  d = 128: BM = 64 with two tensor-memory buffers
// for S/P and dP/dQ, so the MMAs of one query tile overlap the exponentials
// of the next.  d = 64: BM = 128 and one buffer (the dQ MMA would otherwise
// need M = 64).
//
// Q and dO have rings of their own: three Q slots, and for d = 128 two dO
// slots.  The MMA warp issues tile t+1's S^T before tile t's gradient MMAs
// and tile t+1's dP^T after them, so a dO slot is refilled one tile after it
// is released (the dP^T of tile t+1 is needed only once the compute warps
// have finished P_{t+1} and drained dQ_t).
//
// Statistics folded into the MMAs (bf16 kernels without dropout): the
// per-query values LSE2_i and Dvec_i would otherwise be read by every thread
// (one key row each) for every query column, 64 KB of shared-memory
// broadcast per 64-query tile.  Instead each S^T and dP^T product takes one
// more K = 16 step: A = a ones block (128 key rows x 16, columns {0, 1, 2,
// 8, 9, 10} one), B = the query tile's slab (its rows hold a three-way bf16
// split of -LSE2_i / (scale log2 e), resp. -Dvec_i, in columns 0-2, zeros
// elsewhere).  The accumulators then hold S - LSE2/(scale log2 e) and
// dP - Dvec, so P = exp2(acc * scale * log2 e) and dS = P o acc.  The ones
// rows are all equal and each 16-byte half of a row holds the same values,
// so the 32-byte swizzle (which only exchanges the halves of a row) leaves
// the block unchanged.
template <int D_, bool FP16_>
struct BwdCfg {
  static constexpr int D = D_;
  static constexpr bool FP16 = FP16_;
  static constexpr int BN = 128;
  static constexpr int BM = (D == 128) ? 64 : 128;
  static constexpr int NBUF = (D == 128) ? 2 : 1;
  static constexpr bool DQT = (D == 128);  // dQ^T = K^T dS^T (M = d), else dQ = dS K (M = BM)
  static constexpr int QSTAGES = 3;
  static constexpr int DOSTAGES = (D == 128) ? 2 : 3;
  static constexpr int NBOX = D / 64;
  static constexpr int NQB = BM / 64;
  static constexpr int HW = BM / 2;  // query columns per compute warp
  static constexpr int DQW = DQT ? BM : D;  // columns of a dQ block in tensor memory
  static_assert(DQW == 64, "each compute warp drains a 32 x 32 part of the dQ block");
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int DS_BYTES = BN * BM * 2;
  static constexpr int SLAB_BYTES = BM * kSlabRowBytes;  // one tile's statistics slab
  static constexpr int ONES_BYTES = BN * kSlabRowBytes;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_BYTES;
  static constexpr int OFF_Q = OFF_V + KV_BYTES;
  static constexpr int OFF_DO = OFF_Q + QSTAGES * Q_BYTES;
  static constexpr int OFF_DS = OFF_DO + DOSTAGES * Q_BYTES;
  // dQ staging: two 4 KB boxes (32 x 32 fp32, 128-byte swizzle) per drain warp
  static constexpr int DQS_BYTES = 32 * 32 * 4;
  static constexpr int OFF_DQS = OFF_DS + NBUF * DS_BYTES;
  static constexpr int OFF_LSB = OFF_DQS + 8 * DQS_BYTES;  // -LSE2 slabs, one per Q slot
  static constexpr int OFF_DVB = OFF_LSB + QSTAGES * SLAB_BYTES;  // -Dvec slabs, per dO slot
  static constexpr int OFF_ONES = OFF_DVB + DOSTAGES * SLAB_BYTES;
  static constexpr int OFF_LSE = OFF_ONES + ONES_BYTES;  // fp32 LSE2, per Q slot (no fold)
  static constexpr int OFF_DVEC = OFF_LSE + QSTAGES * BM * 4;  // fp32 Dvec, per dO slot
  static constexpr int OFF_BAR = OFF_DVEC + DOSTAGES * BM * 4;
  // barriers
  static constexpr int B_KV = 0;
  static constexpr int B_QFULL = 1;
  static constexpr int B_DOFULL = B_QFULL + QSTAGES;
  static constexpr int B_QEMPTY = B_DOFULL + DOSTAGES;
  static constexpr int B_DOEMPTY = B_QEMPTY + QSTAGES;
  static constexpr int B_SFULL = B_DOEMPTY + DOSTAGES;  // per buffer
  static constexpr int B_DPFULL = B_SFULL + NBUF;
  static constexpr int B_PREADY = B_DPFULL + NBUF;    // 256 arrivals
  static constexpr int B_DSREADY = B_PREADY + NBUF;   // 256 arrivals
  static constexpr int B_DSFREE = B_DSREADY + NBUF;
  static constexpr int B_DQFULL = B_DSFREE + NBUF;
  static constexpr int B_DQFREE = B_DQFULL + NBUF;    // 128 arrivals (the drain warps)
  static constexpr int B_DONE = B_DQFREE + NBUF;
  static constexpr int NBAR = B_DONE + 1;
  static constexpr int OFF_TMEMPTR = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_TMEMPTR + 16 + 1024;
  // tensor memory: dV, dK accumulators; per buffer an S/P block and a dP/dQ block
  static constexpr int TM_DV = 0, TM_DK = D, TM_S = 2 * D, TM_DP = 2 * D + NBUF * BM;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 448;  // 8 compute, producer, MMA, 4 dQ drain warps
  static_assert(TM_DP + NBUF * BM <= TMEM_COLS, "tensor memory");
  static_assert(DQT || D <= BM, "dQ block fits its dP block");
  static_assert(QSTAGES * Q_BYTES >= BN * D * 2, "dK epilogue staging");
  static_assert(DOSTAGES * Q_BYTES >= BN * D * 2, "dV epilogue staging");
  static_assert(OFF_LSB % 1024 == 0 && SLAB_BYTES % 256 == 0, "32-byte swizzle atoms");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <class C, bool ALIBI, bool DROP>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_lse2, const __grid_constant__ CUtensorMap tm_dvec,
                    const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                    const __grid_constant__ CUtensorMap tm_dqacc, const BwdParams pin) {
  constexpr int D = C::D, BN = C::BN, BM = C::BM, NBUF = C::NBUF, QS = C::QSTAGES;
  constexpr int DS = C::DOSTAGES;
  // tm_lse2 / tm_dvec are the slab maps when FOLD, the fp32 row maps otherwise
  constexpr bool FOLD = !C::FP16 && !DROP;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem0 = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem0 - smem_addr(smem_raw));
  auto bar = [&](int i) -> uint32_t { return smem0 + C::OFF_BAR + 8u * i; };
  volatile uint32_t* tmem_ptr_slot = reinterpret_cast<volatile uint32_t*>(smem_gen + C::OFF_TMEMPTR);

  const uint32_t warp = warp_id(), lane = lane_id();
  // earlier key tiles are seen by more queries under a causal mask: heaviest
  // first
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
  // Padded row of this sequence's first query in the Dvec / LSE2 rows and
  // the dQ accumulator (packed layout; the dense layout indexes by batch).
  const long long prow0 = p.cu_q ? packed_row0(sq.q_row0, b) : 0;
  const bool row_store = p.cu_q != nullptr && k0 + BN > p.seqlen_k;

  // Query rows that see any key of [k0, k1).
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

  // Statistics coordinates of tile t: query head, first query row, the row
  // of the statistics arrays ((padded row, head) packed, (row, batch*head)
  // dense) and its column.
  auto tile_stat = [&](int t, int& h, int& q0, int& row, int& xs) {
    h = kvh * group + t / nqb;
    q0 = (qb_lo + t % nqb) * BM;
    row = p.cu_q ? h : b * p.nheads + h;
    xs = (int)prow0 + q0;
  };
  // Q_t (and its LSE2 statistics) into Q slot t % QS.
  auto load_q = [&](int t) -> bool {
    const int slot = t % QS, n = t / QS;
    if (n > 0 && !mbar_wait(bar(C::B_QEMPTY + slot), (n - 1) & 1)) return false;
    int h, q0, row, xs;
    tile_stat(t, h, q0, row, xs);
    mbar_arrive_expect_tx(bar(C::B_QFULL + slot), C::Q_BYTES + (FOLD ? C::SLAB_BYTES : BM * 4));
    for (int bx = 0; bx < C::NBOX; ++bx)
      tma_load_4d(smem0 + C::OFF_Q + slot * C::Q_BYTES + bx * (BM * 128), &tm_q,
                  bar(C::B_QFULL + slot), bx * 64, h, sq.q_row0 + q0, sq.tma_b);
    if constexpr (FOLD)
      tma_load_3d(smem0 + C::OFF_LSB + slot * C::SLAB_BYTES, &tm_lse2, bar(C::B_QFULL + slot), 0,
                  xs, row);
    else
      tma_load_2d(smem0 + C::OFF_LSE + slot * BM * 4, &tm_lse2, bar(C::B_QFULL + slot), xs, row);
    return true;
  };
  // dO_t (and its Dvec statistics) into dO slot t % DS.
  auto load_do = [&](int t) -> bool {
    const int slot = t % DS, n = t / DS;
    if (n > 0 && !mbar_wait(bar(C::B_DOEMPTY + slot), (n - 1) & 1)) return false;
    int h, q0, row, xs;
    tile_stat(t, h, q0, row, xs);
    mbar_arrive_expect_tx(bar(C::B_DOFULL + slot), C::Q_BYTES + (FOLD ? C::SLAB_BYTES : BM * 4));
    for (int bx = 0; bx < C::NBOX; ++bx)
      tma_load_4d(smem0 + C::OFF_DO + slot * C::Q_BYTES + bx * (BM * 128), &tm_do,
                  bar(C::B_DOFULL + slot), bx * 64, h, sq.q_row0 + q0, sq.tma_b);
    if constexpr (FOLD)
      tma_load_3d(smem0 + C::OFF_DVB + slot * C::SLAB_BYTES, &tm_dvec, bar(C::B_DOFULL + slot),
                  0, xs, row);
    else
      tma_load_2d(smem0 + C::OFF_DVEC + slot * BM * 4, &tm_dvec, bar(C::B_DOFULL + slot), xs,
                  row);
    return true;
  };

  // The producer lane initialises the barriers and starts the K, V and
  // first query-tile loads before the block-wide barrier, so that their
  // latency overlaps the tensor-memory allocation and the barrier itself.
  if (warp == 8 && lane == 0) {
    for (int i = 0; i < C::NBAR; ++i) {
      uint32_t count = 1;
      if (i >= C::B_PREADY && i < C::B_DSREADY + NBUF) count = 256;  // compute warps
      if (i >= C::B_DQFREE && i < C::B_DQFREE + NBUF) count = 128;   // drain warps
      mbar_init(bar(i), count);
    }
    fence_barrier_init();
    fence_proxy_async_smem();
    if (nt > 0) {
      mbar_arrive_expect_tx(bar(C::B_KV), 2 * C::KV_BYTES);
      for (int bx = 0; bx < C::NBOX; ++bx) {
        tma_load_4d(smem0 + C::OFF_K + bx * (BN * 128), &tm_k, bar(C::B_KV), bx * 64, kvh,
                    sq.k_row0 + k0, sq.tma_b);
        tma_load_4d(smem0 + C::OFF_V + bx * (BN * 128), &tm_v, bar(C::B_KV), bx * 64, kvh,
                    sq.k_row0 + k0, sq.tma_b);
      }
      load_q(0);  // first use of its slots: no wait
      load_do(0);
    }
  }
  if constexpr (FOLD) {
    // The ones block of the statistics step: 128 rows of 32 bytes, each
    // 16-byte half = bf16 {1, 1, 1, 0, 0, 0, 0, 0}; one half per thread.
    if (warp < 8) {
      st_shared_v4(smem0 + C::OFF_ONES + threadIdx.x * 16, 0x3F803F80u, 0x00003F80u, 0u, 0u);
      fence_proxy_async_smem();
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
      for (int t = 1; t < nt; ++t)  // K, V and tile 0 are on their way
        if (!load_q(t) || !load_do(t)) break;
      for (int t = nt - QS < 0 ? 0 : nt - QS; t < nt; ++t)
        if (!mbar_wait(bar(C::B_QFULL + t % QS), (t / QS) & 1)) break;
      for (int t = nt - DS < 0 ? 0 : nt - DS; t < nt; ++t)
        if (!mbar_wait(bar(C::B_DOFULL + t % DS), (t / DS) & 1)) break;
      mbar_wait(bar(C::B_KV), 0);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the issue loop (its values stay warp-uniform); one
    // elected lane issues each MMA and commit.
    if (nt > 0) {
      constexpr uint32_t idesc_s = idesc_f16(BN, BM, C::FP16, false, false);
      constexpr uint32_t idesc_acc = idesc_f16(BN, D, C::FP16, false, true);
      constexpr uint32_t idesc_dq =
          C::DQT ? idesc_f16(D, BM, C::FP16, true, true) : idesc_f16(BM, D, C::FP16, true, true);
      // K and V stay put: their descriptors (K-major for S^T / dP^T, MN-major
      // K for the dQ MMA) are built once.
      const uint64_t k_kdesc = sdesc_sw128(smem0 + C::OFF_K, 16, 1024);
      const uint64_t v_kdesc = sdesc_sw128(smem0 + C::OFF_V, 16, 1024);
      const uint64_t k_mndesc = sdesc_sw128(smem0 + C::OFF_K, BN * 128, 1024);
      const uint64_t ones_desc = sdesc_sw32(smem0 + C::OFF_ONES, 256);
      // S^T_u = K Q_u^T (- LSE2 / (scale log2 e) when FOLD) into the S block
      // of buffer u % NBUF.
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
        if constexpr (FOLD)
          mma_ss_warp(tmem + C::TM_S + bf * BM, ones_desc,
                      sdesc_sw32(smem0 + C::OFF_LSB + slot * C::SLAB_BYTES, 256), idesc_s, 1u);
        mma_commit_warp(bar(C::B_SFULL + bf));
        return true;
      };
      // dP^T_u = V dO_u^T (- Dvec when FOLD) into the dP block, once tile
      // u - NBUF's dQ left it.
      auto issue_dp = [&](int u) -> bool {
        const int slot = u % DS, bf = u % NBUF, use = u / NBUF;
        const uint64_t do_desc = sdesc_sw128(smem0 + C::OFF_DO + slot * C::Q_BYTES, 16, 1024);
        if (use > 0 && !mbar_wait_warp(bar(C::B_DQFREE + bf), (use - 1) & 1)) return false;
        if (!mbar_wait_warp(bar(C::B_DOFULL + slot), (u / DS) & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int bx = kk / 4, w = kk % 4;
          mma_ss_warp(tmem + C::TM_DP + bf * BM, desc_at(v_kdesc, bx * (BN * 128) + w * 32),
                 desc_at(do_desc, bx * (BM * 128) + w * 32), idesc_s, kk > 0);
        }
        if constexpr (FOLD)
          mma_ss_warp(tmem + C::TM_DP + bf * BM, ones_desc,
                      sdesc_sw32(smem0 + C::OFF_DVB + slot * C::SLAB_BYTES, 256), idesc_s, 1u);
        mma_commit_warp(bar(C::B_DPFULL + bf));
        return true;
      };
      // dV += P^T dO, dK += dS^T Q and tile t's dQ share; then Q and dO of
      // tile t are released.
      auto issue_grads = [&](int t) -> bool {
        const int qslot = t % QS, dslot = t % DS, bf = t % NBUF, use = t / NBUF;
        const uint64_t q_mn = sdesc_sw128(smem0 + C::OFF_Q + qslot * C::Q_BYTES, BM * 128, 1024);
        const uint64_t do_mn = sdesc_sw128(smem0 + C::OFF_DO + dslot * C::Q_BYTES, BM * 128, 1024);
        const uint32_t ds_base = smem0 + C::OFF_DS + bf * C::DS_BYTES;
        const uint64_t ds_mn = sdesc_sw128(ds_base, BN * 128, 1024);
        if (!mbar_wait_warp(bar(C::B_PREADY + bf), use & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk) {
          // P^T from tensor memory: each half of the query columns keeps its
          // packed values at the start of its own score columns.
          const int half = kk / (C::HW / 16), part = kk % (C::HW / 16);
          mma_ts_warp(tmem + C::TM_DV, tmem + C::TM_S + bf * BM + half * C::HW + part * 8,
                 desc_at(do_mn, kk * 2048), idesc_acc, (t > 0 || kk > 0));
        }
        if (!mbar_wait_warp(bar(C::B_DSREADY + bf), use & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk) {
          // dS^T from tensor memory, packed after each half's P^T; Q MN-major
          const int half = kk / (C::HW / 16), part = kk % (C::HW / 16);
          mma_ts_warp(tmem + C::TM_DK,
                      tmem + C::TM_S + bf * BM + half * C::HW + C::HW / 2 + part * 8,
                      desc_at(q_mn, kk * 2048), idesc_acc, (t > 0 || kk > 0));
        }
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          if constexpr (C::DQT)  // dQ^T = K^T dS^T: both operands MN-major
            mma_ss_warp(tmem + C::TM_DP + bf * BM, desc_at(k_mndesc, kk * 2048),
                   desc_at(ds_mn, kk * 2048), idesc_dq, kk > 0);
          else  // dQ = dS K
            mma_ss_warp(tmem + C::TM_DP + bf * BM, desc_at(ds_mn, kk * 2048),
                   desc_at(k_mndesc, kk * 2048), idesc_dq, kk > 0);
        }
        mma_commit_warp(bar(C::B_DQFULL + bf));
        mma_commit_warp(bar(C::B_DSFREE + bf));
        mma_commit_warp(bar(C::B_QEMPTY + qslot));
        mma_commit_warp(bar(C::B_DOEMPTY + dslot));
        return true;
      };
      // Two buffers: tile t+1's S^T goes in before tile t's gradient MMAs
      // and its dP^T after them (the dP block of t+1 is released when the
      // compute warps drain tile t-1's dQ, midway through tile t).  One
      // buffer: tile t first.
      bool ok = mbar_wait_warp(bar(C::B_KV), 0) && issue_s(0) && issue_dp(0);
      for (int t = 0; ok && t < nt; ++t) {
        const bool more = t + 1 < nt;
        if (NBUF == 2 && more && !issue_s(t + 1)) { ok = false; break; }
        if (!issue_grads(t)) { ok = false; break; }
        if (NBUF == 2 && more && !issue_dp(t + 1)) { ok = false; break; }
        if (NBUF == 1 && more && !(issue_s(t + 1) && issue_dp(t + 1))) { ok = false; break; }
      }
      if (ok) mma_commit_warp(bar(C::B_DONE));
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ P, dS
    // Warp w: tensor-memory lane quadrant w % 4 (key rows), query-column half
    // w / 4 (HW columns).
    const int quad = (int)(warp & 3), half = (int)(warp >> 2);
    const int r = quad * 32 + (int)lane;  // key row within the tile == TMEM lane
    const int c0 = half * C::HW;          // first query column of this warp
    const long long j = (long long)k0 + r;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    bool ok = true;
    for (int t = 0; t < nt; ++t) {
      const int qslot = t % QS, dslot = t % DS, bf = t % NBUF, use = t / NBUF;
      const int q0 = (qb_lo + t % nqb) * BM;
      if (!mbar_wait_warp(bar(C::B_SFULL + bf), use & 1)) { ok = false; break; }
      if (!FOLD && !mbar_wait_warp(bar(C::B_QFULL + qslot), (t / QS) & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t s_tmem = tmem + lane_base + C::TM_S + bf * BM + c0;
      float pr[C::HW];
#pragma unroll
      for (int c = 0; c < C::HW; c += 32) {
        uint32_t raw[32];
        tmem_ld32(s_tmem + c, raw);
#pragma unroll
        for (int e = 0; e < 32; ++e) pr[c + e] = __uint_as_float(raw[e]);
      }
      tmem_ld_wait();
      // Whole half visible.  Without the fold, query rows past seqlen_q have
      // LSE2 = +inf (P = 0); with it they are masked here.
      const int qa = q0 + c0;
      const bool full = ((long long)k0 + BN <= p.seqlen_k) &&
                        ((long long)k0 + BN - 1 <= (long long)qa + off + rb) &&
                        ((long long)k0 >= (long long)(qa + C::HW - 1) + off - lb) &&
                        (!FOLD || qa + C::HW <= p.seqlen_q);
      const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
      // positional bias of query column c (ALIBI): bk * |c - bd|, log2 units
      const int hq = kvh * group + t / nqb;  // this tile's query head
      const float bk = ALIBI ? -p.alibi[hq] * 1.4426950408889634f : 0.f;
      const float bd = ALIBI ? (float)(j - off - qa) : 0.f;
      if constexpr (FOLD) {
#pragma unroll
        for (int c = 0; c < C::HW; c += 2) {
          float a0, a1;
          f2_unpack(f2_mul(f2_pack(pr[c], pr[c + 1]), scale2), a0, a1);
          if constexpr (ALIBI) {
            a0 = fmaf(fabsf((float)c - bd), bk, a0);
            a1 = fmaf(fabsf((float)(c + 1) - bd), bk, a1);
          }
          pr[c] = ex2(a0);
          pr[c + 1] = ex2(a1);
        }
      } else {
        const uint32_t lse_addr = smem0 + C::OFF_LSE + (qslot * BM + c0) * 4;
#pragma unroll
        for (int c = 0; c < C::HW; c += 4) {
          float l4[4];
          ld_shared_v4f(lse_addr + c * 4, l4);
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            float a0, a1;
            f2_unpack(f2_fma(f2_pack(pr[c + e], pr[c + e + 1]), scale2, f2_pack(-l4[e], -l4[e + 1])),
                      a0, a1);
            if constexpr (ALIBI) {
              a0 = fmaf(fabsf((float)(c + e) - bd), bk, a0);
              a1 = fmaf(fabsf((float)(c + e + 1) - bd), bk, a1);
            }
            pr[c + e] = ex2(a0);
            pr[c + e + 1] = ex2(a1);
          }
        }
      }
      if (!full) {
#pragma unroll
        for (int c = 0; c < C::HW; ++c) {
          const long long i = (long long)qa + c;
          if (j >= p.seqlen_k || j > i + off + rb || j < i + off - lb ||
              (FOLD && i >= p.seqlen_q))
            pr[c] = 0.f;
        }
      }
      // Dropout: this key's random bytes for the warp's query columns, kw[k]
      // for columns 4k .. 4k + 3.  P^T goes to the dV MMA with dropped
      // elements zeroed (dV's 1 / (1 - p) is applied in the epilogue); pr
      // keeps the undropped P for dS.
      [[maybe_unused]] uint32_t kw[C::HW / 4];
      if constexpr (DROP) {
        const uint32_t bh = (uint32_t)(b * p.nheads + hq);
#pragma unroll
        for (int c = 0; c < C::HW; c += 32) {
          uint32_t part[8];
          dropout_col32(p.drop_seed, p.drop_offset, bh, (uint32_t)j, (uint32_t)(qa + c), part);
#pragma unroll
          for (int k = 0; k < 8; ++k) kw[c / 4 + k] = part[k];
        }
      }
#pragma unroll
      for (int c = 0; c < C::HW; c += 32) {
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          w[e] = pack2<C::FP16>(pr[c + 2 * e], pr[c + 2 * e + 1]);
          if constexpr (DROP)
            w[e] &= dropout_pair_mask(dropout_keep_bits(kw[(c + 2 * e) / 4], e & 1, p.drop_kadd));
        }
        tmem_st16(s_tmem + c / 2, w);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(C::B_PREADY + bf));
      if (!mbar_wait_warp(bar(C::B_DPFULL + bf), use & 1)) { ok = false; break; }
      if (!FOLD && !mbar_wait_warp(bar(C::B_DOFULL + dslot), (t / DS) & 1)) { ok = false; break; }
      tc_fence_after();
      if constexpr (FOLD) {
        // the accumulator holds dP - Dvec: dS = P o acc
#pragma unroll
        for (int c = 0; c < C::HW; c += 32) {
          uint32_t raw[32];
          tmem_ld32(tmem + lane_base + C::TM_DP + bf * BM + c0 + c, raw);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            f2_unpack(f2_mul(f2_pack(pr[c + e], pr[c + e + 1]),
                             f2_pack(__uint_as_float(raw[e]), __uint_as_float(raw[e + 1]))),
                      pr[c + e], pr[c + e + 1]);
        }
      } else {
        const uint32_t dvec_addr = smem0 + C::OFF_DVEC + (dslot * BM + c0) * 4;
#pragma unroll
        for (int c = 0; c < C::HW; c += 32) {
          uint32_t raw[32];
          tmem_ld32(tmem + lane_base + C::TM_DP + bf * BM + c0 + c, raw);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            float d4[4];
            ld_shared_v4f(dvec_addr + (c + e) * 4, d4);
#pragma unroll
            for (int f = 0; f < 4; f += 2) {
              // dS = P * (dP - Dvec), two columns per packed instruction pair;
              // with dropout dP of a kept element is scaled by 1 / (1 - p) and
              // that of a dropped one is 0.
              uint64_t diff;
              if constexpr (DROP) {
                const uint32_t kb = dropout_keep_bits(kw[(c + e) / 4], f / 2, p.drop_kadd);
                const float g0 = __uint_as_float(raw[e + f] & dropout_lo_mask(kb));
                const float g1 = __uint_as_float(raw[e + f + 1] & dropout_hi_mask(kb));
                diff = f2_fma(f2_pack(g0, g1), f2_pack(p.drop_scale, p.drop_scale),
                              f2_pack(-d4[f], -d4[f + 1]));
              } else {
                diff = f2_add(f2_pack(__uint_as_float(raw[e + f]), __uint_as_float(raw[e + f + 1])),
                              f2_pack(-d4[f], -d4[f + 1]));
              }
              f2_unpack(f2_mul(f2_pack(pr[c + e + f], pr[c + e + f + 1]), diff), pr[c + e + f],
                        pr[c + e + f + 1]);
            }
          }
        }
      }
      // dS smem buffer is free once tile t - NBUF's dK and dQ MMAs have read it.
      if (use > 0 && !mbar_wait_warp(bar(C::B_DSFREE + bf), (use - 1) & 1)) { ok = false; break; }
      {
        // dS^T packed into tensor memory after this half's P^T (the A operand
        // of dK += dS^T Q; these score columns were read above), and dS as
        // [key row][query] with 128-byte swizzle, 64 queries per box, in
        // shared memory (an MN-major operand of the dQ product).
        const uint32_t row_addr = smem0 + C::OFF_DS + bf * C::DS_BYTES + r * 128;
#pragma unroll
        for (int c = 0; c < C::HW; c += 32) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) w[e] = pack2<C::FP16>(pr[c + 2 * e], pr[c + 2 * e + 1]);
          tmem_st16(s_tmem + C::HW / 2 + c / 2, w);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            const int col = c0 + c + q8 * 8;
            const int bx = col / 64, chunk = ((col % 64) / 8) ^ (r & 7);
            st_shared_v4(row_addr + bx * (BN * 128) + chunk * 16, w[4 * q8], w[4 * q8 + 1],
                         w[4 * q8 + 2], w[4 * q8 + 3]);
          }
        }
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(C::B_DSREADY + bf));
    }
    // ------------------------------------------------------------ epilogue
    if (ok && nt > 0) ok = mbar_wait_warp(bar(C::B_DONE), 0);
    if (ok && p.acc_f32) {
      // float32 accumulate: this warp's 32 key rows x D/2 head-dim columns
      // of dK (x scale), then of dV, as 32 x 32 boxes through its staging
      // box, each added into the caller's buffer by one TMA reduce-add
      // (rows past seqlen_k are clipped by the tensor map).  A key tile that
      // no query sees adds nothing.
      if (nt > 0) {
        tc_fence_after();
        const int krow = sq.k_row0 + k0 + quad * 32;
        // staging box of this warp in the (now idle) Q slots
        const uint32_t dqs = smem0 + C::OFF_Q + warp * 4096;
        bool staged = false;
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
          const uint32_t src = tmem + lane_base + (which == 0 ? C::TM_DK : C::TM_DV);
          const float mul = which == 0 ? p.softmax_scale : 1.f;
#pragma unroll 1
          for (int c = half * (D / 2); c < (half + 1) * (D / 2); c += 32) {
            uint32_t raw[32];
            tmem_ld32(src + c, raw);
            tmem_ld_wait();
            if (staged) {
              if (lane == 0) bulk_wait_group_read_all();
              __syncwarp();
            }
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4)
              st_shared_v4(dqs + lane * 128 + ((c4 ^ (lane & 7)) << 4),
                           __float_as_uint(__uint_as_float(raw[4 * c4]) * mul),
                           __float_as_uint(__uint_as_float(raw[4 * c4 + 1]) * mul),
                           __float_as_uint(__uint_as_float(raw[4 * c4 + 2]) * mul),
                           __float_as_uint(__uint_as_float(raw[4 * c4 + 3]) * mul));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && k0 + quad * 32 < p.seqlen_k) {
              tma_reduce_add_4d(which == 0 ? &tm_dk : &tm_dv, dqs, c, kvh, krow, sq.tma_b);
              bulk_commit_group();
            }
            staged = true;
          }
        }
      }
    } else if (ok) {
      tc_fence_after();
      // dK (x scale) staged in the Q slots, dV in the dO slots; this warp
      // writes head-dim columns [half * D/2, (half + 1) * D/2) of its rows.
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t src = tmem + lane_base + (which == 0 ? C::TM_DK : C::TM_DV);
        const uint32_t row_addr = smem0 + (which == 0 ? C::OFF_Q : C::OFF_DO) + r * 128;
        const float mul = which == 0 ? p.softmax_scale : (DROP ? p.drop_scale : 1.f);
#pragma unroll 1
        for (int c = half * (D / 2); c < (half + 1) * (D / 2); c += 32) {
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
          if (row_store) {
            if (k0 + r < p.seqlen_k) {
              uint16_t* dst = which == 0 ? p.dk : p.dv;
              store_row32(dst + ((size_t)(sq.k_row0 + k0 + r) * p.nheads_kv + kvh) * D + c, w);
            }
            continue;
          }
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
    named_bar_sync(1, 256);
    if (ok && threadIdx.x == 0 && !row_store && !p.acc_f32) {
      for (int bx = 0; bx < C::NBOX; ++bx) {
        tma_store_4d(&tm_dk, smem0 + C::OFF_Q + bx * (BN * 128), bx * 64, kvh, sq.k_row0 + k0,
                     sq.tma_b);
        tma_store_4d(&tm_dv, smem0 + C::OFF_DO + bx * (BN * 128), bx * 64, kvh, sq.k_row0 + k0,
                     sq.tma_b);
      }
      bulk_commit_group();
    }
    // the dK/dV stores or reduces have read their shared memory before exit
    if (lane == 0) bulk_wait_group_read_all();
  } else if (warp >= 10) {
    // ------------------------------------------------------------ dQ drain
    // Warp w reads tensor-memory lane quadrant w % 4 of each tile's dQ block
    // (64 columns: d = 128 holds dQ^T, lanes = head-dim columns and columns
    // = queries; d = 64 holds dQ, lanes = queries and columns = head-dim),
    // releases the block, stages it as two [query][head-dim] fp32 boxes of
    // 32 x 32 (128-byte swizzle) and adds each into the accumulator with one
    // TMA reduce-add (rows past seqlen_q are clipped by the tensor map).
    const int quad = (int)(warp & 3);
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t dqs = smem0 + C::OFF_DQS + (warp - 10) * 2 * C::DQS_BYTES;
    for (int u = 0; u < nt; ++u) {
      const int bf = u % NBUF;
      if (!mbar_wait_warp(bar(C::B_DQFULL + bf), (u / NBUF) & 1)) break;
      tc_fence_after();
      const int h = kvh * group + u / nqb;
      const int q0 = (qb_lo + u % nqb) * BM;
      uint32_t raw[2][32];
      tmem_ld32(tmem + lane_base + C::TM_DP + bf * BM, raw[0]);
      tmem_ld32(tmem + lane_base + C::TM_DP + bf * BM + 32, raw[1]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar(C::B_DQFREE + bf));
      // the previous tile's reduces have read both boxes (issued a whole
      // tile earlier)
      if (u > 0) {
        if (lane == 0) bulk_wait_group_read_all();
        __syncwarp();
      }
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        const uint32_t box = dqs + hb * C::DQS_BYTES;
        // Box element (row, col) sits at row * 128 + ((col / 4) ^ (row % 8)) * 16 + (col % 4) * 4.
        int qrow, dcol;  // the box origin in (query, head-dim)
        if constexpr (C::DQT) {
          // lane = head-dim column quad*32 + lane; columns = queries q0 + hb*32 + c
#pragma unroll
          for (int c = 0; c < 32; ++c)
            st_shared_f32(box + c * 128 + (((lane >> 2) ^ (c & 7)) << 4) + ((lane & 3) << 2),
                          __uint_as_float(raw[hb][c]));
          qrow = q0 + hb * 32;
          dcol = quad * 32;
        } else {
          // lane = query q0 + quad*32 + lane; columns = head-dim hb*32 + c
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4)
            st_shared_v4(box + lane * 128 + ((c4 ^ (lane & 7)) << 4), raw[hb][4 * c4],
                         raw[hb][4 * c4 + 1], raw[hb][4 * c4 + 2], raw[hb][4 * c4 + 3]);
          qrow = q0 + quad * 32;
          dcol = hb * 32;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && qrow < p.seqlen_q) {
          tma_reduce_add_4d(&tm_dqacc, box, dcol, h, (int)prow0 + qrow, sq.tma_b);
          bulk_commit_group();
        }
      }
    }
    if (lane == 0) bulk_wait_group_read_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace attn
