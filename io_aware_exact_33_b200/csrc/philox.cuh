// philox.cuh - counter-based random bytes for attention dropout.
//
// Generator: Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel random
// numbers: as easy as 1, 2, 3", SC 2011).  A round multiplies counter words
// 0 and 2 by two odd 32-bit constants and builds the next counter from the
// 64-bit products' halves, words 1 and 3 and the round key; the key advances
// by two Weyl increments between rounds.  On the GPU __umulhi gives the high
// half of each product and a plain 32-bit multiply the low half.
//
// Dropout contract (the same on every pass and every program that follows
// it): key = (seed low word, seed high word); score element (b, h, i, j) of
// query row i and key column j takes byte (j mod 4) of output word (i mod 4)
// at counter (j / 4, i / 4, b * H + h, offset), so one generator call covers
// a 4 x 4 block of the score matrix, reachable from a row-per-thread layout
// (forward) and a column-per-thread layout (backward, S^T) alike.  The
// element is dropped iff its byte is below the threshold t = round(256 p) in
// [0, 255]; kept values are scaled by 256 / (256 - t).
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define ATTN_HD __host__ __device__ __forceinline__
#else
#define ATTN_HD inline
#endif

namespace attn {

struct Philox4 {
  uint32_t w[4];
};

ATTN_HD uint32_t philox_mulhi(uint32_t a, uint32_t b) {
#if defined(__CUDA_ARCH__)
  return __umulhi(a, b);
#else
  return (uint32_t)(((uint64_t)a * b) >> 32);
#endif
}

// Ten rounds of Philox4x32 on counter c under key (k0, k1).
ATTN_HD Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0,
                              uint32_t k1) {
  constexpr uint32_t kMul0 = 0xD2511F53u, kMul1 = 0xCD9E8D57u;
  constexpr uint32_t kWeyl0 = 0x9E3779B9u, kWeyl1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = philox_mulhi(kMul0, c0), lo0 = kMul0 * c0;
    const uint32_t hi1 = philox_mulhi(kMul1, c2), lo1 = kMul1 * c2;
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
    k0 += kWeyl0;
    k1 += kWeyl1;
  }
  return Philox4{{c0, c1, c2, c3}};
}

// The 16 random bytes of the 4 x 4 score block whose top-left element is
// (4 * ib, 4 * jb) of head bh = b * H + h: word r holds row 4 ib + r, its
// byte c (bits 8c..8c+7) column 4 jb + c.
ATTN_HD Philox4 dropout_block(uint64_t seed, uint32_t offset, uint32_t bh, uint32_t ib,
                              uint32_t jb) {
  return philox4x32_10(jb, ib, bh, offset, (uint32_t)seed, (uint32_t)(seed >> 32));
}

// Keep factor of one element from its random byte u and threshold t.
ATTN_HD float dropout_factor(uint32_t u, uint32_t t) {
  return u < t ? 0.f : 256.f / (float)(256u - t);
}

// The addend of the keep test below: (256 - t) in both 16-bit lanes.
ATTN_HD uint32_t dropout_kadd(uint32_t t) { return (256u - t) * 0x00010001u; }

#if defined(__CUDACC__)
// ---------------------------------------------------------------- in kernels
// The four lanes of an aligned group (lane & ~3) each hold a row of a 4 x 4
// matrix of words, v[k] = M[lane & 3][k]; afterwards each holds a column,
// v[k] = M[k][lane & 3].  Two exchange stages (partner lane ^ 1, then ^ 2),
// each swapping the off-diagonal halves of 2 x 2 blocks.  All 32 lanes call.
__device__ __forceinline__ void group4_transpose(uint32_t (&v)[4]) {
  const uint32_t L = threadIdx.x & 3u;
#pragma unroll
  for (int k = 0; k < 4; k += 2) {
    const uint32_t send = (L & 1u) ? v[k] : v[k + 1];
    const uint32_t got = __shfl_xor_sync(0xffffffffu, send, 1);
    if (L & 1u) v[k] = got; else v[k + 1] = got;
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const uint32_t send = (L & 2u) ? v[k] : v[k + 2];
    const uint32_t got = __shfl_xor_sync(0xffffffffu, send, 2);
    if (L & 2u) v[k] = got; else v[k + 2] = got;
  }
}

// Forward layout: lane = query row `row` (lanes 4g..4g+3 hold rows with the
// same row / 4).  kw[k] = this row's random bytes for key columns
// j0 + 4k .. j0 + 4k + 3 (byte c = column j0 + 4k + c), k < 4; j0 % 4 == 0.
// Each lane runs the generator for one of the group's four blocks.
__device__ __forceinline__ void dropout_row16(uint64_t seed, uint32_t offset, uint32_t bh,
                                              uint32_t row, uint32_t j0, uint32_t (&kw)[4]) {
  const Philox4 b = dropout_block(seed, offset, bh, row >> 2, (j0 >> 2) + (threadIdx.x & 3u));
#pragma unroll
  for (int k = 0; k < 4; ++k) kw[k] = b.w[k];  // word r = row r of this lane's block
  group4_transpose(kw);                         // kw[k] = my row's word of block k
}

// Backward layout (S^T): lane = key column `j` (lanes 4g..4g+3 hold keys with
// the same j / 4).  kw[k] = this key's random bytes for query rows
// i0 + 4k .. i0 + 4k + 3 (byte r = row i0 + 4k + r), k < 8; i0 % 4 == 0.
// The block's bytes are transposed in registers (word c = column c) before
// the cross-lane transpose.
__device__ __forceinline__ void dropout_col32(uint64_t seed, uint32_t offset, uint32_t bh,
                                              uint32_t j, uint32_t i0, uint32_t (&kw)[8]) {
  const uint32_t rho = threadIdx.x & 3u;
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const Philox4 b = dropout_block(seed, offset, bh, (i0 >> 2) + 4u * s + rho, j >> 2);
    const uint32_t t0 = __byte_perm(b.w[0], b.w[1], 0x5140), t1 = __byte_perm(b.w[0], b.w[1], 0x7362);
    const uint32_t t2 = __byte_perm(b.w[2], b.w[3], 0x5140), t3 = __byte_perm(b.w[2], b.w[3], 0x7362);
    uint32_t v[4] = {__byte_perm(t0, t2, 0x5410), __byte_perm(t0, t2, 0x7632),
                     __byte_perm(t1, t3, 0x5410), __byte_perm(t1, t3, 0x7632)};
    group4_transpose(v);  // v[k] = my key column of block 4s + k
#pragma unroll
    for (int k = 0; k < 4; ++k) kw[4 * s + k] = v[k];
  }
}

// Keep test of two elements whose random bytes are bytes 2q and 2q + 1 of
// `word`: each byte goes to a 16-bit lane, gains 256 - t (bit 8 set iff the
// byte is >= t, no carry between lanes), and a shift by 7 brings that bit to
// the top of bytes 1 and 3.
__device__ __forceinline__ uint32_t dropout_keep_bits(uint32_t word, int q, uint32_t kadd) {
  return (__byte_perm(word, 0u, q ? 0x4342 : 0x4140) + kadd) << 7;
}

// Sign replication of a byte's top bit over the selected result bytes
// (prmt in its default mode, selector nibbles with the high bit set).
template <uint32_t SEL>
__device__ __forceinline__ uint32_t prmt_sign(uint32_t x) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(x), "r"(0u), "n"(SEL));
  return r;
}

// 0xFFFF / 0 in each 16-bit lane: the mask of a packed 16-bit pair.
__device__ __forceinline__ uint32_t dropout_pair_mask(uint32_t keep_bits) {
  return prmt_sign<0xBB99u>(keep_bits);
}
// 0xFFFFFFFF / 0 for the first and the second element of the pair.
__device__ __forceinline__ uint32_t dropout_lo_mask(uint32_t keep_bits) {
  return prmt_sign<0x9999u>(keep_bits);
}
__device__ __forceinline__ uint32_t dropout_hi_mask(uint32_t keep_bits) {
  return prmt_sign<0xBBBBu>(keep_bits);
}
#endif

}  // namespace attn
