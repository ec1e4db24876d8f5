// INT2 group quantiser and dequantiser used by the ledger ("Resumo Técnico: QEvict",
// Metodologia: recoverable INT2 tier; Hierarquia Recuperável: write-once ledger).
//
// One row of D elements is held by a warp, DPL = D/32 consecutive elements per lane, so a
// 16-element group spans LPG = 16/DPL consecutive lanes. Per group, in float32 with
// round-to-nearest-even:
//   s = fp16((max - min) / 3), z = fp16(min), code = clamp(rint((x - z) / s), 0, 3), 0 if s == 0.
// Row layout in a ledger entry: codes [D/4] bytes (element 4j+e in bits 2e..2e+1 of byte j),
// meta [D/16] u32 = fp16 s (low half) | fp16 z (high half).
#pragma once
#include "qe_internal.cuh"

// The parameters of one group from its exact min and max: s = fp16((max - min) / 3) with the
// quotient correctly rounded in float32 (the correction for division by a known constant,
// Markstein; Brisebarre, Muller and Raina: q0 = RN(d * RN(1/3)), r = d - 3 q0 exact with an FMA,
// q = RN(q0 + r * RN(1/3)); checked against IEEE division for every non-negative finite float32
// and +inf, which passes through), z = fp16(min); the float values of s and z and an
// approximate reciprocal of s (0 when s == 0).
struct Int2Group {
  __half sh, zh;
  float s, z, rs;
  __device__ __forceinline__ Int2Group(float mn, float mx) {
    const float d3 = __fsub_rn(mx, mn);
    const float third = 0.333333343267440796f;  // RN(1/3)
    float q3 = __fmul_rn(d3, third);
    q3 = __fmaf_rn(__fmaf_rn(-3.f, q3, d3), third, q3);
    q3 = isinf(d3) ? d3 : q3;
    sh = __float2half_rn(q3);
    zh = __float2half_rn(mn);
    s = __half2float(sh);
    z = __half2float(zh);
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
    rs = s != 0.f ? r : 0.f;
  }
  // code = rint(f32(x - z) / s) clamped to [0, 3]: the quotient is formed with the approximate
  // reciprocal (relative error about 2^-23, far below 1e-3); within 1e-3 of a half-integer the
  // correctly rounded division decides instead, so the result is that of rint of the IEEE
  // quotient in every case. s == 0 gives 0; negative values and NaN convert to 0.
  __device__ __forceinline__ uint32_t code(float x) const {
    const float d = __fsub_rn(x, z);
    float qv = __fmul_rn(d, rs);
    if (fabsf(qv - rintf(qv)) > 0.499f) qv = __fdiv_rn(d, s);
    return min(__float2uint_rn(qv), 3u);
  }
  // Parameters (rs, -z) of the fast code path: q = f32(f32(x - z) * rs), with the approximate
  // reciprocal rs (relative error below 2^-22), is within 2^-20 of the IEEE quotient
  // f32(x - z) / s for q < 4, and stays within (-0.5, 3.5) for every x of the group when
  // |min - z| * rs < 0.45. Groups outside that bound (or with s subnormal or infinite in fp16,
  // or z infinite) get -1 in place of rs: the exact path decides. s == 0 gives rs = 0, so every
  // q is 0.
  __device__ __forceinline__ float2 fast_params(float mn) const {
    const bool ok = (s == 0.f || (s >= 0x1p-14f && s <= 65504.f)) && fabsf(z) <= 65504.f &&
                    fabsf(__fsub_rn(mn, z)) * rs < 0.45f;
    return make_float2(ok ? rs : -1.f, -z);
  }
  __device__ __forceinline__ uint32_t meta() const {
    return static_cast<uint32_t>(__half_as_ushort(sh)) | (static_cast<uint32_t>(__half_as_ushort(zh)) << 16);
  }
};

// code = clamp(rint(f32(x - z) / s), 0, 3) by IEEE division; 0 when s == 0 (the definition the
// fast path below falls back on).
__device__ __forceinline__ uint32_t int2_code_exact(float x, float s, float z) {
  if (s == 0.f) return 0u;
  return min(__float2uint_rn(__fdiv_rn(__fsub_rn(x, z), s)), 3u);
}

// The 16 codes of one group, element e at bits 2e of n, from its elements as eight pairs of
// 16-bit values (e2[i] holds elements 2i, 2i + 1) and fast parameters p = (rs, -z), rs >= 0.
// Each q = f32(f32(x - z) * rs) is rounded to an integer by adding 1.5 * 2^23: the sum's bits are
// 0x4B400000 + rint(q) (ties to even, q in (-0.5, 3.5)), so the codes accumulate by shifted
// adds of the raw bits, less the same sum of the constant part. Returns the mask of elements
// whose q lies within 2^-16 of a half-integer (bit e), where q could round the other way than
// the exact quotient (they differ by less than 2^-20): those take the exact path.
template <typename T>
__device__ __forceinline__ uint32_t int2_group_codes_fast(const uint32_t (&e2)[8], float2 p, uint32_t& n) {
  constexpr float kMagic = 12582912.f;  // 1.5 * 2^23, bits 0x4B400000
  constexpr float kNear = 0.5f - 0x1p-16f;
  constexpr uint32_t kBias = [] {
    uint32_t b = 0u;
    for (int e = 0; e < 16; ++e) b += 0x4B400000u << (2 * e);
    return b;
  }();
  const float2 r2 = make_float2(p.x, p.x), nz2 = make_float2(p.y, p.y);
  uint32_t acc = 0u, near = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 x = make_float2(Elem<T>::lo(e2[i]), Elem<T>::hi(e2[i]));
    const float2 q = __fmul2_rn(__fadd2_rn(x, nz2), r2);
    const float2 t = __fadd2_rn(q, make_float2(kMagic, kMagic));
    const float2 e = __ffma2_rn(q, make_float2(-1.f, -1.f), __fadd2_rn(t, make_float2(-kMagic, -kMagic)));
    near |= (fabsf(e.x) > kNear ? 1u : 0u) << (2 * i);
    near |= (fabsf(e.y) > kNear ? 1u : 0u) << (2 * i + 1);
    acc += (__float_as_uint(t.x) << (4 * i)) + (__float_as_uint(t.y) << (4 * i + 2));
  }
  n = acc - kBias;
  return near;
}

template <int DPL>
struct Int2Row {
  static constexpr int LPG = 16 / DPL;  // lanes per 16-element group

  // Quantise the lane's DPL values. Returns the lane's codes packed at bits 2e, and the
  // group's (s, z) as a u32 in *meta (valid in every lane).
  static __device__ __forceinline__ uint32_t quantize(const float (&x)[DPL], uint32_t* meta) {
    float mn = x[0], mx = x[0];
#pragma unroll
    for (int e = 1; e < DPL; ++e) {
      mn = fminf(mn, x[e]);
      mx = fmaxf(mx, x[e]);
    }
#pragma unroll
    for (int o = 1; o < LPG; o <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const Int2Group q(mn, mx);
    uint32_t bits = 0;
#pragma unroll
    for (int e = 0; e < DPL; ++e) bits |= q.code(x[e]) << (2 * e);
    *meta = q.meta();
    return bits;
  }

  // Write the lane's codes (from quantize) into a row of D/4 bytes. All lanes must call.
  static __device__ __forceinline__ void store_codes(uint8_t* row, uint32_t bits, int lane) {
    if (DPL == 4) {
      row[lane] = static_cast<uint8_t>(bits);
    } else {  // DPL == 2: two lanes share a byte
      const uint32_t other = __shfl_down_sync(0xffffffffu, bits, 1);
      if ((lane & 1) == 0) row[lane >> 1] = static_cast<uint8_t>(bits | (other << 4));
    }
  }

  // The lane's DPL codes from a row of D/4 bytes, packed at bits 2e.
  static __device__ __forceinline__ uint32_t load_codes(const uint8_t* row, int lane) {
    if (DPL == 4) return row[lane];
    return (row[lane >> 1] >> (4 * (lane & 1))) & 0xFu;
  }

  static __device__ __forceinline__ int group_of(int lane) { return lane / LPG; }
};

__device__ __forceinline__ float meta_scale(uint32_t m) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(m & 0xffffu)));
}
__device__ __forceinline__ float meta_zero(uint32_t m) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(m >> 16)));
}
