// hq_lattice.cuh -- nearest-point decoders and bit-stripping for the E8, D4, A2 and Z lattices
// ("Lattice Quantization", Methodology step 2; "Bit-Stripping", step 3), device side.
//
// Closest-point rules after Conway & Sloane, "Fast quantizing and decoding algorithms for lattice
// quantizers and codes" (IEEE T-IT 28(2), 1982), in binary32 without contraction:
//   a = rint(u) via the 1.5*2^23 addition (exact for |u| < 2^22, which the per-tile RMS scaling
//   and the step range guarantee), e = a - u (exact, never -0), "toward u" = +1 when e < 0;
//   argmax / argmin of |e| compare max(|e|, 2^-63), ties to the lowest index.
#pragma once

#include "hq_common.cuh"

namespace hq {

constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
constexpr float kTiny = 1.0842021724855044e-19f;  // 2^-63
constexpr float kA2K = 1.15470053837925153f;      // RN(2/sqrt(3))

__device__ __forceinline__ float rint_magic(float u, int32_t& ai)
{
    const float t = __fadd_rn(u, kMagic);
    ai = __float_as_int(t) - __float_as_int(kMagic);
    return __fadd_rn(t, -kMagic);
}

__device__ __forceinline__ float clamp_tiny(float v) { return v < kTiny ? kTiny : v; }

// D4 = {v in Z^4, sum even}; v = the nearest point.
__device__ __forceinline__ void q_d4(const float (&u)[4], int32_t (&v)[4])
{
    float e[4];
    int32_t sum = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float r = rint_magic(u[i], v[i]);
        e[i] = __fadd_rn(r, -u[i]);
        sum += v[i];
    }
    if (sum & 1) {
        int j = 0;
        float best = clamp_tiny(fabsf(e[0]));
#pragma unroll
        for (int i = 1; i < 4; ++i) {
            const float c = clamp_tiny(fabsf(e[i]));
            if (c > best) { best = c; j = i; }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (i == j) v[i] += (e[i] < 0.0f) ? 1 : -1;
    }
}

// E8 = D8 u (D8 + 1/2): v = twice the nearest point.  The coset choice compares
// |u-A|^2 - |u-B|^2 = sum(|e| - 1/4) + [A fixed](1 - 2 max|e|) - [B fixed](2 min|e|) in binary32
// as D = ((S - 2) + cA) - cB, S the pairwise sum of |e|; B only when D > 0.
__device__ __forceinline__ void q_e8(const float (&u)[8], int32_t (&v)[8])
{
    float e[8], ae[8];
    int32_t a[8];
    int32_t sumA = 0, nonneg = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float r = rint_magic(u[i], a[i]);
        e[i] = __fadd_rn(r, -u[i]);
        ae[i] = fabsf(e[i]);
        sumA += a[i];
        nonneg += (e[i] < 0.0f) ? 0 : 1;
    }
    const int parA = sumA & 1;
    const int parB = (sumA - nonneg) & 1;
    const float S = __fadd_rn(__fadd_rn(__fadd_rn(ae[0], ae[1]), __fadd_rn(ae[2], ae[3])),
                              __fadd_rn(__fadd_rn(ae[4], ae[5]), __fadd_rn(ae[6], ae[7])));
    int jA = 0, mB = 0;
    float emax = clamp_tiny(ae[0]), emin = emax;
#pragma unroll
    for (int i = 1; i < 8; ++i) {
        const float c = clamp_tiny(ae[i]);
        if (c > emax) { emax = c; jA = i; }
        if (c < emin) { emin = c; mB = i; }
    }
    const float cA = parA ? __fadd_rn(1.0f, -__fmul_rn(2.0f, emax)) : 0.0f;
    const float cB = parB ? __fmul_rn(2.0f, emin) : 0.0f;
    const float D = __fadd_rn(__fadd_rn(__fadd_rn(S, -2.0f), cA), -cB);
    if (!(D > 0.0f)) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            int32_t ai = a[i];
            if (parA && i == jA) ai += (e[i] < 0.0f) ? 1 : -1;
            v[i] = 2 * ai;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int32_t toward = (e[i] < 0.0f) ? 1 : -1;
            int32_t vi = 2 * a[i] + toward;
            if (parB && i == mB) vi -= 2 * toward;
            v[i] = vi;
        }
    }
}

// A2 with minimum distance 1 in (P, Q) = (2 u0, u1 K); the even point when |eP| + 3|eQ| <= 1.
__device__ __forceinline__ void q_a2(const float (&u)[2], int32_t (&v)[2])
{
    const float P = __fmul_rn(2.0f, u[0]);
    const float Q = __fmul_rn(u[1], kA2K);
    const float hP = __fmul_rn(P, 0.5f), hQ = __fmul_rn(Q, 0.5f);
    int32_t aP, aQ;
    const float rP = rint_magic(hP, aP), rQ = rint_magic(hQ, aQ);
    const float eP = __fadd_rn(rP, -hP), eQ = __fadd_rn(rQ, -hQ);
    const float E = __fadd_rn(fabsf(eP), __fmul_rn(3.0f, fabsf(eQ)));
    if (E <= 1.0f) {
        v[0] = 2 * aP;
        v[1] = 2 * aQ;
    } else {
        v[0] = 2 * aP + ((eP < 0.0f) ? 1 : -1);
        v[1] = 2 * aQ + ((eQ < 0.0f) ? 1 : -1);
    }
}

template <int LAT>
struct Lat;
template <>
struct Lat<HQ_Z> { static constexpr int d = 1; };
template <>
struct Lat<HQ_A2> { static constexpr int d = 2; };
template <>
struct Lat<HQ_D4> { static constexpr int d = 4; };
template <>
struct Lat<HQ_E8> { static constexpr int d = 8; };

// nearest point of one block: u[d] -> integer embedding v[d]
template <int LAT>
__device__ __forceinline__ void quantize_block(const float* u, int32_t* v)
{
    if constexpr (LAT == HQ_Z) {
        rint_magic(u[0], v[0]);
    } else if constexpr (LAT == HQ_A2) {
        const float uu[2] = {u[0], u[1]};
        int32_t vv[2];
        q_a2(uu, vv);
        v[0] = vv[0]; v[1] = vv[1];
    } else if constexpr (LAT == HQ_D4) {
        const float uu[4] = {u[0], u[1], u[2], u[3]};
        int32_t vv[4];
        q_d4(uu, vv);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = vv[i];
    } else {
        float uu[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) uu[i] = u[i];
        int32_t vv[8];
        q_e8(uu, vv);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = vv[i];
    }
}

// bit-stripping of one block: integer embedding v[d] -> d symbols (+ the E8 coset bit)
template <int LAT>
__device__ __forceinline__ uint32_t strip_block(const int32_t* v, int32_t* s)
{
    if constexpr (LAT == HQ_Z) {
        s[0] = v[0];
        return 0u;
    } else if constexpr (LAT == HQ_A2) {
        s[0] = v[0];
        s[1] = (v[1] - (v[0] & 1)) >> 1;
        return 0u;
    } else if constexpr (LAT == HQ_D4) {
        const int32_t p = (v[0] + v[1] + v[2]) & 1;
        s[0] = v[0]; s[1] = v[1]; s[2] = v[2];
        s[3] = (v[3] - p) >> 1;
        return 0u;
    } else {
        const int32_t c = v[0] & 1;
        int32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = (v[i] - c) >> 1;
        const int32_t p = (w[0] + w[1] + w[2] + w[3] + w[4] + w[5] + w[6]) & 1;
#pragma unroll
        for (int i = 0; i < 7; ++i) s[i] = w[i];
        s[7] = (w[7] - p) >> 1;
        return (uint32_t)c;
    }
}

// inverse of strip_block: symbols (+ coset bit) -> integer embedding
template <int LAT>
__device__ __forceinline__ void unstrip_block(const int32_t* s, uint32_t c, int32_t* v)
{
    if constexpr (LAT == HQ_Z) {
        v[0] = s[0];
    } else if constexpr (LAT == HQ_A2) {
        v[0] = s[0];
        v[1] = 2 * s[1] + (s[0] & 1);
    } else if constexpr (LAT == HQ_D4) {
        const int32_t p = (s[0] + s[1] + s[2]) & 1;
        v[0] = s[0]; v[1] = s[1]; v[2] = s[2];
        v[3] = 2 * s[3] + p;
    } else {
        const int32_t p = (s[0] + s[1] + s[2] + s[3] + s[4] + s[5] + s[6]) & 1;
#pragma unroll
        for (int i = 0; i < 7; ++i) v[i] = 2 * s[i] + (int32_t)c;
        v[7] = 2 * (2 * s[7] + p) + (int32_t)c;
    }
}

// KV dither for D4 block `blk` of token (bh, s): U uniform on the Voronoi cell of D4
// ("Subtractive Dither", Methodology step 4).  r = 2 (w >> 8) 2^-24 is uniform on [0,2)^4, a union
// of D4 cells (2Z^4 is a sublattice of D4); U = r - Q_D4(r).
__device__ __forceinline__ void dither_d4(uint64_t seed, uint32_t bh, uint64_t s, uint32_t blk, float (&U)[4])
{
    const uint4 w = philox4x32_10(make_uint4((uint32_t)s, bh, 0x80000000u | blk, (uint32_t)(s >> 32)),
                                  (uint32_t)seed, (uint32_t)(seed >> 32));
    float r[4];
    r[0] = __fmul_rn(2.0f, __fmul_rn((float)(w.x >> 8), 5.9604644775390625e-08f));
    r[1] = __fmul_rn(2.0f, __fmul_rn((float)(w.y >> 8), 5.9604644775390625e-08f));
    r[2] = __fmul_rn(2.0f, __fmul_rn((float)(w.z >> 8), 5.9604644775390625e-08f));
    r[3] = __fmul_rn(2.0f, __fmul_rn((float)(w.w >> 8), 5.9604644775390625e-08f));
    int32_t q[4];
    q_d4(r, q);
#pragma unroll
    for (int i = 0; i < 4; ++i) U[i] = __fadd_rn(r[i], -(float)q[i]);
}

}  // namespace hq
