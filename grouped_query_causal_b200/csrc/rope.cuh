// rope.cuh -- RoPE angle evaluation shared by the prefill and decode kernels.
//
// RoPE ("Qwen3系列1-理论基础&真实结构" D2-2; "深入剖析Qwen3模型架构" 3.1.2 and 3.4.1):
// pair i = (x[2i], x[2i+1]) of a head vector is rotated counter-clockwise by
// phi_i = pos * theta_i:  (a, b) -> (a cos phi - b sin phi, a sin phi + b cos phi),
// theta_i = base^(-2i/D).  Variants: the rotate-half pairing (x[i], x[i + D/2]) with the
// same angles, and frequency tables scaled for longer contexts (linear, NTK-aware, YaRN),
// which the host computes into RopeFreqs.
#pragma once
#include <cstdint>

namespace gqa {

constexpr int kHeadDim = 128;
constexpr int kPairs = kHeadDim / 2;

// theta_i for i = 0 .. D/2-1, evaluated on the host in double precision.
struct RopeFreqs {
    double inv_freq[kPairs];
};

constexpr int kPairAdjacent = 0;   // (x[2i], x[2i+1])
constexpr int kPairHalf = 1;       // (x[i], x[i + D/2])

// A RoPE variant as the kernels use it: frequencies, pairing, and the factor the
// attention logits are multiplied by (1 except for YaRN's temperature).
struct RopeSpec {
    RopeFreqs rf;
    int pairing;
    float logit_mult;
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

// RoPE of one head vector spread over a warp, lane l holding (already normed) elements
// 4l .. 4l+3 in a[0..3], rotated in place to position pos.  Adjacent pairs stay inside a
// lane; with the rotate-half pairing element e meets e +- D/2 in lane l ^ 16, at frequency
// (4l + k) mod D/2.  Every lane of the warp must call it with the same pairing.
__device__ __forceinline__ void rope_warp4(float (&a)[4], int pos, const RopeFreqs &rf, int pairing, int lane) {
    if (pairing == kPairAdjacent) {
        float c0, s0, c1, s1;
        rope_cos_sin(pos, rf.inv_freq[2 * lane], c0, s0);
        rope_cos_sin(pos, rf.inv_freq[2 * lane + 1], c1, s1);
        const float y0 = a[0] * c0 - a[1] * s0, y1 = a[0] * s0 + a[1] * c0;
        const float y2 = a[2] * c1 - a[3] * s1, y3 = a[2] * s1 + a[3] * c1;
        a[0] = y0;
        a[1] = y1;
        a[2] = y2;
        a[3] = y3;
    } else {
        const float sign = lane < 16 ? -1.0f : 1.0f;   // first half: a c - b s; second: a c + b s
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float b = __shfl_xor_sync(0xffffffffu, a[k], 16);
            float c, s;
            rope_cos_sin(pos, rf.inv_freq[4 * (lane & 15) + k], c, s);
            a[k] = fmaf(sign * b, s, a[k] * c);
        }
    }
}

}  // namespace gqa
