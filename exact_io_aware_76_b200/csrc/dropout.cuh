// Attention dropout: the keep mask and how warps share its random words.
//
// The pages name dropout only as the `dropout_p` argument of flash_attn_func (page "Flash Attention — 長い系列を
// 扱う Transformer の学習と推論を速くする", Workflow 2, Step 2). The mask definition used here:
//   t = floor(256 dropout_p + 1/2) (0..255); element (i, j) of head number bh = b * H + h is kept iff byte
//   (j mod 4) of word (i mod 4) of Philox4x32-10(counter = (i / 4, j / 4, bh, offset), key = (seed lo, seed hi))
//   is >= t; kept probabilities are scaled by 1 / (1 - t / 256).
// One generator call thus covers a 4 x 4 block of (query, key) elements. Both kernels regenerate it: the forward
// thread owns a query row, the backward compute thread owns a key row, so four lanes (four rows of one block)
// each generate one block of a run of four and then exchange words with two shuffle stages.
#pragma once
#include <stdint.h>

namespace fa {

// Philox4x32 with 10 rounds (Salmon, Moraes, Dror, Shaw: "Parallel random numbers: as easy as 1, 2, 3", SC 2011).
// A round takes the 64-bit products of words 0 and 2 with the two round multipliers and returns
// (hi(M1*c2) ^ c1 ^ k0, lo(M1*c2), hi(M0*c0) ^ c3 ^ k1, lo(M0*c0)); between rounds the key advances by the two
// Weyl constants (32-bit fractions of the golden ratio and of sqrt(3) - 1).
__device__ __forceinline__ void philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0,
                                              uint32_t k1, uint32_t w[4]) {
  constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u, kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += kW0;
      k1 += kW1;
    }
    const uint32_t hi0 = __umulhi(kM0, c0), lo0 = kM0 * c0;
    const uint32_t hi1 = __umulhi(kM1, c2), lo1 = kM1 * c2;
    c0 = hi1 ^ c1 ^ k0;
    c1 = lo1;
    c2 = hi0 ^ c3 ^ k1;
    c3 = lo0;
  }
  w[0] = c0;
  w[1] = c1;
  w[2] = c2;
  w[3] = c3;
}

// Within each group of four lanes (4a .. 4a+3) every lane holds four words w[0..3]; afterwards lane 4a+r holds
// in w[k] the word r that lane 4a+k held. Two butterfly stages: lanes differing in bit 0 swap the words whose
// index differs from their own lane in bit 0, then the same for bit 1. All 32 lanes must take part.
__device__ __forceinline__ void quad_exchange(uint32_t w[4]) {
  const uint32_t lane = threadIdx.x & 31u;
  const bool b0 = lane & 1u, b1 = lane & 2u;
#pragma unroll
  for (int k = 0; k < 4; k += 2) {
    const uint32_t send = b0 ? w[k] : w[k + 1];
    const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, 1);
    w[k] = b0 ? recv : w[k];
    w[k + 1] = b0 ? w[k + 1] : recv;
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const uint32_t send = b1 ? w[k] : w[k + 2];
    const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, 2);
    w[k] = b1 ? recv : w[k];
    w[k + 2] = b1 ? w[k + 2] : recv;
  }
}

// Transpose a 4 x 4 byte matrix held as four words (word = row, byte 0 = column 0): afterwards word c holds
// column c (its byte r = the old byte c of word r).
__device__ __forceinline__ void byte_transpose4(uint32_t w[4]) {
  const uint32_t t0 = __byte_perm(w[0], w[1], 0x5140), t1 = __byte_perm(w[0], w[1], 0x7362);
  const uint32_t t2 = __byte_perm(w[2], w[3], 0x5140), t3 = __byte_perm(w[2], w[3], 0x7362);
  w[0] = __byte_perm(t0, t2, 0x5410);
  w[1] = __byte_perm(t0, t2, 0x7632);
  w[2] = __byte_perm(t1, t3, 0x5410);
  w[3] = __byte_perm(t1, t3, 0x7632);
}

// 1 if byte c of w is >= t.
__device__ __forceinline__ bool keep_byte(uint32_t w, int c, uint32_t t) { return ((w >> (8 * c)) & 0xffu) >= t; }

}  // namespace fa
