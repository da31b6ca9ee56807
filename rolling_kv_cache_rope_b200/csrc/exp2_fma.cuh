// exp2 on the FMA pipe (no MUFU), used for part of the softmax exponentials.
#pragma once

#include <cuda_runtime.h>

namespace rkv {

// 2^x for a pair of floats, on the FMA pipe instead of MUFU (the attention
// softmax is bound by MUFU throughput, so a fraction of its exponentials go
// this way).  Valid for x < 127.5; x below -126 is clamped to -126, which
// returns about 2^-126 (the cubic's value at 0 is just under 1, so the
// exponent sum stays >= 0 only from -126 up).
// j = round(x) by adding 1.5*2^23; 2^(x-j) from the cubic fitted by
// fit_exp2_poly.py (relative error < 8e-5 on [-1/2, 1/2]); 2^j added to the
// exponent field: the low 9 bits of 1.5*2^23's pattern are zero, so
// (bits(x + 1.5*2^23) << 23) == j << 23 modulo 2^32.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 t = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));
  const float2 r = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
  const float2 f = __ffma2_rn(r, make_float2(-1.f, -1.f), x);
  float2 q = __ffma2_rn(make_float2(0x1.c34958p-5f, 0x1.c34958p-5f), f, make_float2(0x1.f0da64p-3f, 0x1.f0da64p-3f));
  q = __ffma2_rn(q, f, make_float2(0x1.62f51ap-1f, 0x1.62f51ap-1f));
  q = __ffma2_rn(q, f, make_float2(0x1.fff6bp-1f, 0x1.fff6bp-1f));
  return make_float2(__int_as_float(__float_as_int(q.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(q.y) + (__float_as_int(t.y) << 23)));
}

}  // namespace rkv
