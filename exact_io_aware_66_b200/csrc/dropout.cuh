// Dropout keep decisions on the GPU.
//
// "How FlashAttention Actually Works" (section "The GPU Memory Wall: HBM vs. SRAM") places dropout
// on the softmax matrix, between the softmax and the product with V. The kernels apply inverted
// dropout there without ever storing a mask: each decision is recomputed from a counter-based
// generator wherever an entry of P is formed, in the forward and again in the backward.
//
// Generator: Philox4x32-10 as defined by Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers:
// As Easy as 1, 2, 3" (SC'11), section 4: a 4-word counter and 2-word key; each of the ten rounds
// multiplies counter words 0 and 2 by 0xD2511F53 and 0xCD9E8D57 into 64-bit products and mixes
// their halves with words 1 and 3 and the key; the key then advances by 0x9E3779B9, 0xBB67AE85.
//
// Mapping (this library's own): for query head bh, query row i and key j,
//   counter = (j >> 2, i >> 2, bh, offset), key = (seed low word, seed high word),
//   byte    = bits [8 (j & 3), 8 (j & 3) + 8) of output word (i & 3),
//   keep    = byte >= p8 (the drop probability is p8 / 256; kept entries scale by 256/(256-p8)).
// One generator call thus serves a 4 x 4 block of (query, key) entries; the four lanes of a
// quad (four consecutive rows of a tile) share its calls through shuffles.
#pragma once

#include <cstdint>

namespace fa {

struct DropoutParams {
  uint32_t seed_lo, seed_hi;  // Philox key
  uint32_t offset;            // counter word 3
  uint32_t add4;              // (256 - p8) in each byte: the byte compare's addend
  float keep_scale;           // 256 / (256 - p8)
};

__device__ __forceinline__ void philox4x32_10(uint32_t (&c)[4], uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c[0];
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c[2];
    const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c[1] ^ k0;
    const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c[3] ^ k1;
    c[0] = n0;
    c[1] = static_cast<uint32_t>(p1);
    c[2] = n2;
    c[3] = static_cast<uint32_t>(p0);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
}

// 4 x 4 transpose across the lanes of a quad: lane s of the quad holds a row a[0..3]; afterwards
// lane r holds column r (a[s] = the former a[r] of lane s). Two butterfly steps of shuffles.
__device__ __forceinline__ void quad_transpose(uint32_t (&a)[4], int lane) {
  {
    const bool hi = lane & 1;
    const uint32_t r0 = __shfl_xor_sync(0xffffffffu, hi ? a[0] : a[1], 1);
    const uint32_t r1 = __shfl_xor_sync(0xffffffffu, hi ? a[2] : a[3], 1);
    if (hi) { a[0] = r0; a[2] = r1; } else { a[1] = r0; a[3] = r1; }
  }
  {
    const bool hi = lane & 2;
    const uint32_t r0 = __shfl_xor_sync(0xffffffffu, hi ? a[0] : a[2], 2);
    const uint32_t r1 = __shfl_xor_sync(0xffffffffu, hi ? a[1] : a[3], 2);
    if (hi) { a[0] = r0; a[1] = r1; } else { a[2] = r0; a[3] = r1; }
  }
}

// 4 x 4 byte transpose within one thread: byte r of t[c] = byte c of w[r].
__device__ __forceinline__ void byte_transpose(const uint32_t (&w)[4], uint32_t (&t)[4]) {
  const uint32_t a_lo = __byte_perm(w[0], w[1], 0x5140), a_hi = __byte_perm(w[0], w[1], 0x7362);
  const uint32_t b_lo = __byte_perm(w[2], w[3], 0x5140), b_hi = __byte_perm(w[2], w[3], 0x7362);
  t[0] = __byte_perm(a_lo, b_lo, 0x5410);
  t[1] = __byte_perm(a_lo, b_lo, 0x7632);
  t[2] = __byte_perm(a_hi, b_hi, 0x5410);
  t[3] = __byte_perm(a_hi, b_hi, 0x7632);
}

// Per byte x of `bytes`: 0xff in that byte if x >= p8, else 0x00. The decision is the carry-out
// of the byte-wise sum x + (256 - p8), computed without cross-byte carries (add the low 7 bits,
// take the majority of the two top bits and the carry into bit 7), then widened from bit 7 to
// the whole byte (0x01 * 0xff stays inside its byte).
__device__ __forceinline__ uint32_t keep_bytes(uint32_t bytes, uint32_t add4) {
  const uint32_t s7 = (bytes & 0x7f7f7f7fu) + (add4 & 0x7f7f7f7fu);
  const uint32_t carry = ((bytes & add4) | ((bytes | add4) & s7)) & 0x80808080u;
  return (carry >> 7) * 0xffu;
}

// Mask for a packed bf16 pair from the keep bytes of entries (2H, 2H+1) of `kb`: 0xffff in
// each half whose entry is kept.
template <int H>
__device__ __forceinline__ uint32_t pair_mask(uint32_t kb) {
  return __byte_perm(kb, 0u, H == 0 ? 0x1100 : 0x3322);
}

// All-ones / all-zeros mask from the keep byte of entry E of `kb`.
template <int E>
__device__ __forceinline__ uint32_t elem_mask(uint32_t kb) {
  return __byte_perm(kb, 0u, 0x1111 * E);
}

}  // namespace fa
