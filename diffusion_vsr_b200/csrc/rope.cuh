// Rotary position embedding (RoPE) of q and k, applied where the kernels read
// them: the cache append (k tiles in shared memory), the draft mask (q before
// its block means) and the attention (Q tiles in shared memory).
//
// RoPE is named by the reading notes "FlashVSR: Towards Real-time
// Diffusion-Based Streaming Video Super Resolution" (背景, 关键设计 3) as the
// relative position code whose periodicity the local window contains; the
// pages give no layout.  The layout used here: each adjacent pair of
// dimensions (2i, 2i+1) of a 128-dim head turns by an angle pos * w_i; the 64
// pairs form three axis bands, pairs [0, 22) over the latent frame (its
// position in the stream), [22, 43) over the token row, [43, 64) over the
// token column; inside a band of n pairs w_i = base^(-i/n).  cos and sin are
// evaluated in fp64 and rounded to fp32; the rotation is taken in fp32 with
// one rounding per product and per sum (no fused multiply-add), and the result
// rounded to bf16 (nearest even): the rotated values are the bf16 inputs of
// everything after.
#pragma once

#include <cstdint>
#include <cuda.h>

namespace lcsa {

constexpr int kRopePairsT = 22;  // time band: pairs [0, 22)
constexpr int kRopePairsY = 21;  // row band: pairs [22, 43)
constexpr int kRopeFirstY = 22;
constexpr int kRopeFirstX = 43;  // column band: pairs [43, 64)

// Axis of a pair (0 time, 1 row, 2 column) and its index inside the band.
__device__ __forceinline__ int rope_axis(int pair) { return pair < kRopeFirstY ? 0 : (pair < kRopeFirstX ? 1 : 2); }

// w of a pair, fp64.
__device__ __forceinline__ double rope_freq(int pair, float base) {
    const int axis = rope_axis(pair);
    const int i = axis == 0 ? pair : (axis == 1 ? pair - kRopeFirstY : pair - kRopeFirstX);
    const int n = axis == 0 ? kRopePairsT : kRopePairsY;
    return pow(static_cast<double>(base), -static_cast<double>(i) / static_cast<double>(n));
}

// Largest stream / token position a rotation may use: |angle| < 2^20.
constexpr int kRopeMaxPos = 1 << 20;

// sin and cos of x, |x| < 2^20, in fp64, by Cody and Waite's method
// ("Software Manual for the Elementary Functions", 1980): reduce
// x = k (pi/2) + r with pi/2 split into three parts, the first two of 33
// significant bits so that k times them is exact for |k| < 2^20 (the three
// parts below are the leading digits of pi/2 taken 33 bits at a time, and the
// rest), then the Maclaurin series of sin and cos on |r| <= pi/4 up to the
// r^17 and r^18 terms (the remainders are below 1e-19), then the quadrant.
__device__ __forceinline__ void rope_sincos(double x, double &s, double &c) {
    constexpr double kHalfPi1 = 0x1.921fb544p+0;        // pi/2, first 33 bits
    constexpr double kHalfPi2 = 0x1.0b4611a6p-34;       // next 33 bits
    constexpr double kHalfPi3 = 0x1.3198a2e037073p-69;  // the rest, rounded
    constexpr double kTwoOverPi = 0.63661977236758134;
    const double k = rint(x * kTwoOverPi);
    double r = fma(-k, kHalfPi1, x);
    r = fma(-k, kHalfPi2, r);
    r = fma(-k, kHalfPi3, r);
    const double r2 = r * r;
    // sin r = r + r^3 P(r^2), P = -1/3! + r^2/5! - r^4/7! + ... + r^14/17!
    double ps = 1.0 / 355687428096000.0;       //  1/17!
    ps = fma(ps, r2, -1.0 / 1307674368000.0);  // -1/15!
    ps = fma(ps, r2, 1.0 / 6227020800.0);      //  1/13!
    ps = fma(ps, r2, -1.0 / 39916800.0);       // -1/11!
    ps = fma(ps, r2, 1.0 / 362880.0);          //  1/9!
    ps = fma(ps, r2, -1.0 / 5040.0);           // -1/7!
    ps = fma(ps, r2, 1.0 / 120.0);             //  1/5!
    ps = fma(ps, r2, -1.0 / 6.0);              // -1/3!
    const double sr = fma(r * r2, ps, r);
    // cos r = 1 + r^2 Q(r^2), Q = -1/2! + r^2/4! - r^4/6! + ... - r^16/18!
    double pc = -1.0 / 6402373705728000.0;     // -1/18!
    pc = fma(pc, r2, 1.0 / 20922789888000.0);  //  1/16!
    pc = fma(pc, r2, -1.0 / 87178291200.0);    // -1/14!
    pc = fma(pc, r2, 1.0 / 479001600.0);       //  1/12!
    pc = fma(pc, r2, -1.0 / 3628800.0);        // -1/10!
    pc = fma(pc, r2, 1.0 / 40320.0);           //  1/8!
    pc = fma(pc, r2, -1.0 / 720.0);            // -1/6!
    pc = fma(pc, r2, 1.0 / 24.0);              //  1/4!
    pc = fma(pc, r2, -0.5);                    // -1/2!
    const double cr = fma(r2, pc, 1.0);
    const int q = static_cast<int>(k) & 3;
    s = q == 0 ? sr : (q == 1 ? cr : (q == 2 ? -sr : -cr));
    c = q == 0 ? cr : (q == 1 ? -sr : (q == 2 ? -cr : sr));
}

// (cos, sin) of pos * w, evaluated in fp64, rounded to fp32.
__device__ __forceinline__ float2 rope_cs(int pos, double w) {
    double s, c;
    rope_sincos(static_cast<double>(pos) * w, s, c);
    return make_float2(__double2float_rn(c), __double2float_rn(s));
}

// Rotates the bf16 pair (a, b) of a bf16x2 word (a in the low half) by (c, s):
// (a c - b s, a s + b c) in fp32, each product and sum rounded once, then
// rounded to bf16x2.
__device__ __forceinline__ uint32_t rope_rotate(uint32_t word, float c, float s) {
    const float a = __uint_as_float(word << 16);
    const float b = __uint_as_float(word & 0xFFFF0000u);
    const float ra = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
    const float rb = __fadd_rn(__fmul_rn(a, s), __fmul_rn(b, c));
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(rb), "f"(ra));  // first source -> upper half
    return r;
}

}  // namespace lcsa
