// RoPE angle for both arithmetic paths (the bf16 projection epilogues and the fp32 kernels).
#pragma once
#include <cuda_runtime.h>

namespace mla {

// cos and sin of the RoPE angle pos * theta^(-2 pair / 64) (pair < 32, the decoupled 64-wide
// rotary part).  The angle (up to ~1.3e5 rad at 128K positions) is formed in double precision
// and reduced modulo 2 pi with 2 pi split into a double head and a tail (Cody and Waite's
// two-constant reduction); what is left, |r| <= pi, goes to the float sincos.  Absolute error
// ~2e-7 at any position up to 2^31 - 1.
__device__ __forceinline__ float2 rope_cs(float theta, int pair, int pos) {
  constexpr double kTwoPiHi = 6.283185307179586;       // nearest double to 2 pi
  constexpr double kTwoPiLo = 2.4492935982947064e-16;  // 2 pi - kTwoPiHi
  constexpr double kInvTwoPi = 0.15915494309189535;
  const double inv_freq = pow(static_cast<double>(theta), -2.0 * pair / 64.0);
  const double a = static_cast<double>(pos) * inv_freq;
  const double k = rint(a * kInvTwoPi);
  const double r = fma(-k, kTwoPiLo, fma(-k, kTwoPiHi, a));
  float sn, cs;
  sincosf(static_cast<float>(r), &sn, &cs);
  return make_float2(cs, sn);
}

}  // namespace mla
