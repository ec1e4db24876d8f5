// Layout of an INT2 ledger entry, arranged for the warp-level tensor cores.
//
// "Resumo Técnico: QEvict", Metodologia 2 (the recoverable INT2 tier stays readable by
// attention) and Hierarquia Recuperável (the write-once ledger). The values stored are those
// of the group quantiser in int2.cuh (2-bit codes, fp16 scale and zero per 16 consecutive
// head-dim elements of one token); only their placement differs from the row-major form that
// qe_int2_quantize and qe_ledger_read use.
//
// An entry of a window of w tokens is w/16 blocks of 16 tokens, 16*D bytes each (128 bytes per
// token at D = 128, the same as the row-major form):
//   KC [32 lanes][D/32 u32]  K codes, each lane's words in the order its mma.sync B fragments
//                            take them (S = Q K^T, query heads as rows, tokens as columns)
//   VC [32 lanes][D/32 u32]  V codes, in the order of the A fragments of O^T = V^T P^T
//   KS [D/16][16]            fp16 K scales, group-major, tokens in pair order (below)
//   KZ [16 tokens][D/16]     fp16 K zeros, token-major
//   VS [D/16][16]            fp16 V scales, group-major, fragment order
//   VZ [D/16][16]            fp16 V zeros, group-major, fragment order
// Pair order of a group's 16 tokens: position 2r + j holds token r + 8j, so one 4-byte load
// gives lane (r, t) the scales of the two tokens of its score rows. Fragment order: position
// 4t + j holds token 2t, 2t+1, 8+2t, 9+2t for j = 0..3, so one 8-byte load gives lane (r, t)
// the pairs its P^T fragments need.
//
// Code placement. Word j of a lane holds the codes of groups 2j (bytes 0 and 2) and 2j+1
// (bytes 1 and 3); within a 16-bit half, bits [2i, 2i+1] of each byte feed register i of the
// decoder, which takes them with a mask (x & (0x00030003 << 2i), after a shift by 8 for the odd
// group): a code c at bit 2i of a half is the fp16 subnormal c * 4^i * 2^-24, an exact operand
// of a 16-bit MMA. The powers 4^i are undone on the other operand or on the accumulator.
//   K, lane 4*r + t (r = token row 0..7, t = 0..3), group g, e = half, i = 2*tb + h:
//     token r + 8*tb, element 16g + 2t + e + 8h
//   V, lane 4*r + t (r = element row 0..7), group g, e = half, i = 2*rh + kh:
//     token 2t + e + 8*kh, element 16g + r + 8*rh
#pragma once
#include "qe_internal.cuh"

template <int D>
struct Int2Block {
  static constexpr int G8 = D / 16;          // INT2 groups per row
  static constexpr int WPL = D / 32;         // code words per lane and per K or V
  static constexpr int KC = 0;
  static constexpr int VC = 4 * D;
  static constexpr int KS = 8 * D;
  static constexpr int KZ = 10 * D;
  static constexpr int VS = 12 * D;
  static constexpr int VZ = 14 * D;
  static constexpr int BYTES = 16 * D;

  // position of token t (0..15) in the fragment order / pair order of a group-major array
  static __host__ __device__ __forceinline__ int fpos(int t) {
    return 4 * ((t & 7) >> 1) + (t & 1) + 2 * (t >> 3);
  }
  static __host__ __device__ __forceinline__ int ppos(int t) { return 2 * (t & 7) + (t >> 3); }

  // (lane, word, bit) of the K / V code of token t (0..15), element d (0..D-1)
  static __host__ __device__ __forceinline__ void kpos(int t, int d, int& lane, int& word, int& bit) {
    const int g = d >> 4, r = d & 15;
    lane = 4 * (t & 7) + ((r >> 1) & 3);
    word = g >> 1;
    bit = 16 * (r & 1) + 8 * (g & 1) + 2 * ((r >> 3) + 2 * (t >> 3));
  }
  static __host__ __device__ __forceinline__ void vpos(int t, int d, int& lane, int& word, int& bit) {
    const int g = d >> 4, r = d & 15;
    lane = 4 * (r & 7) + ((t & 7) >> 1);
    word = g >> 1;
    bit = 16 * (t & 1) + 8 * (g & 1) + 2 * ((t >> 3) + 2 * (r >> 3));
  }

  // The packed words of a block (all lanes, words[lane * WPL + j]) -> byte n (0 .. 16*D/4 - 1)
  // of the row-major codes (nat[t * D/4 + d/4], element d in bits 2(d%4)).
  template <bool V>
  static __device__ __forceinline__ uint8_t unpack_byte(const uint32_t* words, int n) {
    const int t = n / (D / 4), d0 = 4 * (n % (D / 4));
    uint32_t b = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      int ln, wd, bt;
      if (!V) kpos(t, d0 + e, ln, wd, bt);
      else vpos(t, d0 + e, ln, wd, bt);
      b |= ((words[ln * WPL + wd] >> bt) & 3u) << (2 * e);
    }
    return static_cast<uint8_t>(b);
  }
};
