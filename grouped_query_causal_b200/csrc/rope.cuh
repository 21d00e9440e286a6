// rope.cuh -- RoPE angle evaluation shared by the prefill and decode kernels.
//
// RoPE ("Qwen3系列1-理论基础&真实结构" D2-2; "深入剖析Qwen3模型架构" 3.1.2 and 3.4.1):
// pair i = (x[2i], x[2i+1]) of a head vector is rotated counter-clockwise by
// phi_i = pos * theta^(-2i/D):  (a, b) -> (a cos phi - b sin phi, a sin phi + b cos phi).
#pragma once
#include <cstdint>

namespace gqa {

constexpr int kHeadDim = 128;
constexpr int kPairs = kHeadDim / 2;

// theta^(-2i/D) for i = 0 .. D/2-1, evaluated on the host in double precision.
struct RopeFreqs {
    double inv_freq[kPairs];
};

// cos/sin of pos * inv_freq.  The angle (up to ~3.3e4 rad at the longest contexts) is
// formed and reduced modulo 2*pi in double, so the single-precision sincosf only ever
// sees |r| <= pi and the result keeps float accuracy at every position.
__device__ __forceinline__ void rope_cos_sin(int pos, double inv_freq, float &c, float &s) {
    const double kTwoPi = 6.283185307179586476925286766559;
    const double kInvTwoPi = 0.15915494309189533576888376337251;
    const double a = static_cast<double>(pos) * inv_freq;
    const double k = rint(a * kInvTwoPi);
    const float r = static_cast<float>(fma(-k, kTwoPi, a));
    sincosf(r, &s, &c);
}

}  // namespace gqa
