// decode.cuh -- in-register codebook decode of packed 4-bit weights into
// bf16 MMA operands ("Receipts-driven engineering", opening paragraph and
// results table row "Prefill after the v6 register-LUT mainloop rewrite":
// the codebook is decoded in registers inside the GEMM mainloop).
//
// For one scale block the 16 possible decoded values are fixed, so the
// decoder first builds the block's table T[q] = bf16_rn(code[q] * scale)
// (exactly the weight the CPU decoder produces) and then looks codes up with
// byte permutes, no memory access per weight:
//   - T is split into a low-byte plane and a high-byte plane, each as two
//     8-entry halves (q < 8, q >= 8) held in two registers;
//   - `prmt` with the packed codes (bit 3 masked) as selector picks the
//     byte of four codes at once from each half; a second `prmt` with a
//     selector built from bit 3 picks the half; a third interleaves the
//     planes into bf16x2 words.
// Cost: 21 integer ops per 8 weights plus ~32 per table.
#pragma once

#include "common.cuh"

namespace gbw {

struct Planes {
  uint32_t la0, la1, lb0, lb1;  // low bytes of T[0..3], T[4..7], T[8..11], T[12..15]
  uint32_t ha0, ha1, hb0, hb1;  // high bytes
};

// R[j] = T[2j] | T[2j+1] << 16  ->  byte planes.
__device__ __forceinline__ Planes make_planes(const uint32_t (&R)[8]) {
  Planes p;
  p.la0 = prmt(R[0], R[1], 0x6420u);
  p.la1 = prmt(R[2], R[3], 0x6420u);
  p.lb0 = prmt(R[4], R[5], 0x6420u);
  p.lb1 = prmt(R[6], R[7], 0x6420u);
  p.ha0 = prmt(R[0], R[1], 0x7531u);
  p.ha1 = prmt(R[2], R[3], 0x7531u);
  p.hb0 = prmt(R[4], R[5], 0x7531u);
  p.hb1 = prmt(R[6], R[7], 0x7531u);
  return p;
}

// NF4 table of one 64-block: T[q] = bf16_rn(NF4[q] * a).
__device__ __forceinline__ Planes nf4_planes(float a) {
  // QLoRA NF4 levels
  constexpr float c0 = -1.0f, c1 = -0.6961928009986877f,
                  c2 = -0.5250730514526367f, c3 = -0.39491748809814453f,
                  c4 = -0.28444138169288635f, c5 = -0.18477343022823334f,
                  c6 = -0.09105003625154495f, c7 = 0.0f,
                  c8 = 0.07958029955625534f, c9 = 0.16093020141124725f,
                  c10 = 0.24611230194568634f, c11 = 0.33791524171829224f,
                  c12 = 0.44070982933044434f, c13 = 0.5626170039176941f,
                  c14 = 0.7229568362236023f, c15 = 1.0f;
  uint32_t R[8];
  R[0] = pack_bf16x2(__fmul_rn(c0, a), __fmul_rn(c1, a));
  R[1] = pack_bf16x2(__fmul_rn(c2, a), __fmul_rn(c3, a));
  R[2] = pack_bf16x2(__fmul_rn(c4, a), __fmul_rn(c5, a));
  R[3] = pack_bf16x2(__fmul_rn(c6, a), __fmul_rn(c7, a));
  R[4] = pack_bf16x2(__fmul_rn(c8, a), __fmul_rn(c9, a));
  R[5] = pack_bf16x2(__fmul_rn(c10, a), __fmul_rn(c11, a));
  R[6] = pack_bf16x2(__fmul_rn(c12, a), __fmul_rn(c13, a));
  R[7] = pack_bf16x2(__fmul_rn(c14, a), __fmul_rn(c15, a));
  return make_planes(R);
}

// MXFP4 table of one 32-block with e8m0 scale byte s:
// T[q] = bf16_rn(e2m1(q) * 2^(s-127)).  For 2 <= s <= 252 every non-zero
// entry is a normal bf16 and scaling by 2^(s-127) is an integer add to the
// exponent field; other scales (and NaN = 0xFF) take the fp32 route.
__device__ __forceinline__ Planes mxfp4_planes(uint32_t s) {
  uint32_t R[8];
  if (s >= 2u && s <= 252u) {
    const int32_t d = (int32_t)s - 127;
    const uint32_t dh = (uint32_t)d << 23;              // high half only
    const uint32_t dd = ((uint32_t)d << 7) + dh;        // both halves
    // bf16 of e2m1 codes: 0, .5, 1, 1.5, 2, 3, 4, 6 and their negatives
    R[0] = 0x3F000000u + dh;  // 0 stays +0
    R[1] = 0x3FC03F80u + dd;
    R[2] = 0x40404000u + dd;
    R[3] = 0x40C04080u + dd;
    R[4] = 0xBF008000u + dh;  // -0 stays -0
    R[5] = 0xBFC0BF80u + dd;
    R[6] = 0xC040C000u + dd;
    R[7] = 0xC0C0C080u + dd;
  } else {
    const float f = (s == 0xFFu) ? __int_as_float(0x7FC00000)
                  : (s == 0u ? __int_as_float(0x00400000)
                             : __int_as_float((int)(s << 23)));
    const float m[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      R[j] = pack_bf16x2(__fmul_rn(m[2 * j], f), __fmul_rn(m[2 * j + 1], f));
      R[4 + j] = pack_bf16x2(__fmul_rn(-m[2 * j], f), __fmul_rn(-m[2 * j + 1], f));
    }
  }
  return make_planes(R);
}

// Decodes one packed 32-bit word (8 codes, 8 consecutive k) into 4 bf16x2
// words (k order).  kNF4Order: even k in the high nibble (bitsandbytes);
// otherwise even k in the low nibble (OCP / gpt-oss bytes).
template <bool kNF4Order>
__device__ __forceinline__ void decode_word(uint32_t P, const Planes& t,
                                            uint32_t* o) {
  constexpr uint32_t sel0 = kNF4Order ? 0x4051u : 0x5140u;
  constexpr uint32_t sel1 = kNF4Order ? 0x6273u : 0x7362u;
  const uint32_t s = P & 0x77777777u;
  const uint32_t f = ((P >> 1) & 0x44444444u) | 0x32103210u;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t sh = h ? (s >> 16) : s;
    const uint32_t fh = h ? (f >> 16) : f;
    const uint32_t L = prmt(prmt(t.la0, t.la1, sh), prmt(t.lb0, t.lb1, sh), fh);
    const uint32_t H = prmt(prmt(t.ha0, t.ha1, sh), prmt(t.hb0, t.hb1, sh), fh);
    o[2 * h] = prmt(L, H, sel0);
    o[2 * h + 1] = prmt(L, H, sel1);
  }
}

}  // namespace gbw
