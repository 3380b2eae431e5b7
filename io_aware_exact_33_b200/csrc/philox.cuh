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

}  // namespace attn
