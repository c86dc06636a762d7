// In-register dequantization of the frozen 4-bit base into BF16 pairs.
//
// INT4 (two's-complement nibble q, BF16 group scale s): w = bf16(q * s).
//   The nibble u = q & 15 is turned into the exact BF16 integer 136 + q by
//   writing (u ^ 8) into the mantissa of 128.0 (bits 0x4300); subtracting
//   136.0 gives q exactly and one BF16 multiply rounds q * s once.
// MXFP4 (E2M1 code, E8M0 group exponent X): w = bf16(e2m1 * 2^(X-127)).
//   Placing the sign at bit 15 and the three magnitude bits at bits 8..6
//   makes the BF16 number e2m1 * 2^-126 (exact, code 1 lands on a
//   subnormal); multiplying by 2^(X-1) (X <= 128), or by 2^126 and then
//   2^(X-127) (X > 128), gives the scaled value, exact unless it overflows.
//
// Element order: byte i of a packed row holds element 2i (low nibble) and
// element 2i+1 (high nibble); outputs are BF16 pairs (2p, 2p+1).
#pragma once

#include "common.cuh"

namespace moeq {

// Each step is written as one explicit PTX instruction: left to the compiler,
// masks followed by multiplies get rewritten into longer shift/add sequences
// once the known-zero bits are visible, roughly doubling the instruction count.

// Selector of prmt(w, w >> 4, sel): output bytes {w.byte[p], -, (w>>4).byte[p], -};
// the high byte of each half is masked away afterwards.
__device__ __forceinline__ uint32_t pair_select(int p) {
  return static_cast<uint32_t>(p | (p << 4) | ((4 + p) << 8) | ((4 + p) << 12));
}

// Selector of prmt(lo, hi, sel): output bytes {lo.byte[p], 0, hi.byte[p], 0}. The
// zero bytes use prmt's sign-replicate mode on a byte whose top bit is clear.
__device__ __forceinline__ uint32_t pair_select_zero(int p) {
  return static_cast<uint32_t>(p | (0x8 << 4) | ((4 + p) << 8) | (0x8 << 12));
}

// w >> 4 as a multiply-high, so the shift runs on the FMA pipe and leaves the
// integer ALU pipe (which carries the byte permutes and logic ops) free.
__device__ __forceinline__ uint32_t shr4(uint32_t w) {
  uint32_t r;
  asm("mul.hi.u32 %0, %1, 268435456;" : "=r"(r) : "r"(w));
  return r;
}

__device__ __forceinline__ uint32_t and_xor(uint32_t a, uint32_t b, uint32_t c) {  // (a & b) ^ c
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t and_b32(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("and.b32 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t mul_lo(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.lo.u32 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t bf16x2_sub_rn(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t bf16x2_mul_rn(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// 8 INT4 codes of one 32-bit word -> 4 BF16 pairs, scale pair s2 = {s, s}.
__device__ __forceinline__ void dequant8_int4(uint32_t w, uint32_t s2, uint32_t (&o)[4]) {
  const uint32_t odd = shr4(w);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    // {136 + q_even, 136 + q_odd}, then (v - 136) * s
    const uint32_t t = and_xor(prmt(w, odd, pair_select(p)), 0x000F000Fu, 0x43084308u);
    o[p] = bf16x2_mul_rn(bf16x2_sub_rn(t, 0x43084308u), s2);
  }
}

struct MxScale {
  uint32_t a, b;   // BF16 pairs
  bool two;        // apply b after a
};

// E8M0 exponent X -> multipliers turning (e2m1 * 2^-126) into e2m1 * 2^(X-127).
__device__ __forceinline__ MxScale mx_scale(uint32_t X) {
  MxScale s;
  if (X <= 128u) {
    const uint32_t b = (X + 126u) << 7;          // 2^(X-1)
    s.a = b | (b << 16);
    s.b = 0x3F803F80u;
    s.two = false;
  } else {
    s.a = 0x7E807E80u;                           // 2^126
    const uint32_t b = (X == 255u) ? 0x7FC0u : (X << 7);   // 2^(X-127) or NaN
    s.b = b | (b << 16);
    s.two = true;
  }
  return s;
}

// 8 E2M1 codes of one 32-bit word -> 4 BF16 pairs; TWO selects the second
// multiply (exponents above 128).
template <bool TWO>
__device__ __forceinline__ void dequant8_mxfp4(uint32_t w, const MxScale& s, uint32_t (&o)[4]) {
  const uint32_t lo = and_b32(w, 0x0F0F0F0Fu);          // even codes, one per byte
  const uint32_t hi = and_b32(shr4(w), 0x0F0F0F0Fu);    // odd codes
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const uint32_t t = prmt(lo, hi, pair_select_zero(p));   // {c_even, 0, c_odd, 0}
    // c * 0x1040 = (c << 6) + (c << 12) without carries: magnitude to bits
    // 8..6, sign to bit 15 (bits 24..22 and 31 for the upper half); the mask
    // drops the spare copies.
    const uint32_t v = and_b32(mul_lo(t, 0x1040u), 0x81C081C0u);
    uint32_t r = bf16x2_mul_rn(v, s.a);
    if constexpr (TWO) r = bf16x2_mul_rn(r, s.b);
    o[p] = r;
  }
}

// Dequantizes 32 consecutive elements (16 packed bytes, one quantization
// group) into 16 BF16 pairs. FMT: MOE_W_INT4_G32_BF16 or MOE_W_MXFP4_G32_E8M0;
// `scale_bits` holds the BF16 scale bits or the E8M0 exponent.
template <int FMT>
__device__ __forceinline__ void dequant32(const uint4& pk, uint32_t scale_bits, uint32_t (&o)[16]) {
  const uint32_t words[4] = {pk.x, pk.y, pk.z, pk.w};
  if constexpr (FMT == MOE_W_INT4_G32_BF16) {
    const uint32_t s2 = scale_bits | (scale_bits << 16);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t q[4];
      dequant8_int4(words[i], s2, q);
#pragma unroll
      for (int j = 0; j < 4; ++j) o[4 * i + j] = q[j];
    }
  } else {
    // One branch per 32-element group: the second multiply is needed only for
    // exponents above 128, which real weights never use.
    const MxScale s = mx_scale(scale_bits);
    if (!s.two) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t q[4];
        dequant8_mxfp4<false>(words[i], s, q);
#pragma unroll
        for (int j = 0; j < 4; ++j) o[4 * i + j] = q[j];
      }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t q[4];
        dequant8_mxfp4<true>(words[i], s, q);
#pragma unroll
        for (int j = 0; j < 4; ++j) o[4 * i + j] = q[j];
      }
    }
  }
}

}  // namespace moeq
