// Online-softmax pieces shared by the attention kernels (block list and variable-length tiles):
// the row max and the exponentiation of one S row held in registers by its softmax thread.
#pragma once
#include "ptx.cuh"

namespace bsa {

// Largest P a block may produce before the reference max of its rows moves.
constexpr float kMaxP = 1073741824.0f;  // 2^30
constexpr float kMaxLog2P = 30.f;

// Row max of BS fp32 scores (three-input max, four independent chains).
template <int BS>
__device__ __forceinline__ float row_max(const uint32_t (&s)[BS]) {
    float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int e = 0; e < BS; e += 2)
        m4[(e >> 1) & 3] = fmax3f(m4[(e >> 1) & 3], __uint_as_float(s[e]), __uint_as_float(s[e + 1]));
    return fmax3f(fmaxf(m4[0], m4[1]), m4[2], m4[3]);
}

// P = 2^(s * sl2 - m) for a row of BS scores: bf16 pairs into pk, returns the row sum.  Three of
// every four pairs go through the SFU (ex2), one through the FMA-pipe polynomial; bf16 packing
// runs on the integer pipe.  The SFU gives +inf above 2^128, which the sum shows; the polynomial
// is only valid below 2^127, so the largest exponent it was given is returned in xpoly.
template <int BS>
__device__ __forceinline__ float exp_row(const uint32_t (&s)[BS], float sl2, float m,
                                         uint32_t (&pk)[BS / 2], float &xpoly) {
    const float2 sl2v = make_float2(sl2, sl2);
    const float2 nmv = make_float2(-m, -m);
    float2 lacc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float xp = -INFINITY;
#pragma unroll
    for (int e = 0; e < BS; e += 2) {
        const float2 xv = __ffma2_rn(make_float2(__uint_as_float(s[e]), __uint_as_float(s[e + 1])),
                                     sl2v, nmv);
        float2 pv;
        if ((e & 6) == 6) {
            pv = exp2_poly2(xv);
            xp = fmax3f(xp, xv.x, xv.y);
        } else {
            pv.x = ex2(xv.x);
            pv.y = ex2(xv.y);
        }
        lacc[(e >> 1) & 1] = __fadd2_rn(lacc[(e >> 1) & 1], pv);
        pk[e >> 1] = pack_bf16_int(pv.x, pv.y);
    }
    xpoly = xp;
    return (lacc[0].x + lacc[0].y) + (lacc[1].x + lacc[1].y);
}

}  // namespace bsa
