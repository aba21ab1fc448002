// hq_lattice.cuh -- nearest-point decoders and bit-stripping for the E8, D4, A2 and Z lattices
// ("Lattice Quantization", Methodology step 2; "Bit-Stripping", step 3), device side.
//
// Closest-point rules after Conway & Sloane, "Fast quantizing and decoding algorithms for lattice
// quantizers and codes" (IEEE T-IT 28(2), 1982), in binary32 without contraction:
//   a = rint(u) via the 1.5*2^23 addition (exact for |u| < 2^22, which the per-tile RMS scaling
//   and the step range guarantee), e = a - u (exact, never -0), "toward u" = +1 when e < 0;
//   argmax / argmin of |e| with ties to the lowest index.  D4 compares exact 32-bit keys (bits of
//   |e| << 2 | index).  E8's eight coordinates need three index bits, so its keys are
//   max(|e|, 2^-31) bits << 4 | index << 1 | sign of e: the bits of |e| in [2^-31, 1/2] all start
//   with 0011, so the shift drops nothing that orders them, and one integer max / min returns the
//   value, the lowest tied index and the sign together.  Where the 2^-31 floor could change the
//   outcome (a fix-up among rounding errors below 2^-31), and where two cosets (E8, A2) come within
//   a band of a tie that covers the rounding of the shortcut formula, the plain rule runs instead:
//   exact argmax / argmin and both candidates' squared distances in binary32, summed in coordinate
//   order.  Both paths therefore return the point the plain definition returns.
#pragma once

#include "hq_common.cuh"

namespace hq {

constexpr float kMagic = 12582912.0f;         // 1.5 * 2^23
constexpr uint32_t kTinyBits = 0x30000000u;   // 2^-31
constexpr float kA2K = 1.15470053837925153f;  // RN(2/sqrt(3))
// Width of the band around a coset tie in which the plain distance comparison decides.  The
// shortcut value of |u-A|^2 - |u-B|^2 (E8) is within 1.4e-6 of the exact one and the plain
// binary32 distance difference within 3.4e-6 (u^2 units); outside 2^-16 both have the exact sign.
// For A2 the shortcut |eP| + 3|eQ| - 1 and the plain (dE - dO)/4 are both within 1e-6.
constexpr float kTieBand = 1.52587890625e-05f;  // 2^-16

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

__device__ __forceinline__ float rint_magic(float u, int32_t& ai)
{
    const float t = __fadd_rn(u, kMagic);
    ai = __float_as_int(t) - __float_as_int(kMagic);
    return __fadd_rn(t, -kMagic);
}

// argmax key of coordinate i of a d-block: clamped |e| bits, then index (d-1-i, so the lowest
// index wins ties), then the sign of e
__device__ __forceinline__ uint32_t max_key(float e, int i, int d)
{
    const uint32_t eb = __float_as_uint(e);
    const uint32_t mag = max(eb & 0x7FFFFFFFu, kTinyBits);
    return (mag << 4) | ((uint32_t)(d - 1 - i) << 1) | (eb >> 31);
}
__device__ __forceinline__ float key_value(uint32_t key) { return __uint_as_float((key >> 4) | kTinyBits); }

// D4 = {v in Z^4, sum even}; v = the nearest point: round, and if the sum is odd move the
// coordinate with the largest rounding error one step toward u.  |e| <= 1/2, so the bits of |e|
// fit in 30 bits and bits(e) << 2 is |e|'s bits << 2 (the sign shifts out): with the index in
// the two low bits one integer max is the exact argmax with the lowest index on ties, for every
// |e| down to 0.  The sign of the chosen coordinate's e is picked out afterwards.
__device__ __forceinline__ void q_d4(const float (&u)[4], int32_t (&v)[4])
{
    int32_t sum = 0;
    uint32_t kmax = 0;
    float e[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float r = rint_magic(u[i], v[i]);
        sum += v[i];
        e[i] = __fadd_rn(r, -u[i]);
        kmax = max(kmax, (__float_as_uint(e[i]) << 2) | (uint32_t)(3 - i));
    }
    const int j = 3 - (int)(kmax & 3u);
    const float ej = j == 0 ? e[0] : (j == 1 ? e[1] : (j == 2 ? e[2] : e[3]));
    const int32_t delta = (sum & 1) ? (ej < 0.0f ? 1 : -1) : 0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (i == j) v[i] += delta;
}

// The plain E8 coset choice from the rounding errors e (doubled coordinates z = 2u, where a coset A
// point is 2a (+2 toward z at the fixed coordinate) and a coset B point 2a + toward (-2 toward at
// the fixed coordinate), so z - p = -2e - c exactly): exact argmax / argmin of |e| with the lowest
// index on ties, squared distances summed in coordinate order in binary32, A on ties.  Returns
// isB | fix << 1 | (delta + 1) << 4, delta the move of the fixed coordinate of w.  Rarely taken.
static __device__ __forceinline__ uint32_t e8_plain_choice(const float e0, const float e1, const float e2, const float e3,
                                                        const float e4, const float e5, const float e6, const float e7,
                                                        const uint32_t parA, const uint32_t parB)
{
    const float e[8] = {e0, e1, e2, e3, e4, e5, e6, e7};
    int j = 0, m = 0;
    float bmax = fabsf(e[0]), bmin = bmax;
    float ej = e[0], em = e[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) {
        const float a = fabsf(e[i]);
        if (a > bmax) {
            bmax = a;
            j = i;
            ej = e[i];
        }
        if (a < bmin) {
            bmin = a;
            m = i;
            em = e[i];
        }
    }
    float dA = 0.0f, dB = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float t = e[i] < 0.0f ? 1.0f : -1.0f;
        const float cA = (parA && i == j) ? 2.0f * t : 0.0f;
        const float cB = (parB && i == m) ? -t : t;
        const float xA = __fadd_rn(__fmul_rn(-2.0f, e[i]), -cA);
        const float xB = __fadd_rn(__fmul_rn(-2.0f, e[i]), -cB);
        dA = __fadd_rn(dA, __fmul_rn(xA, xA));
        dB = __fadd_rn(dB, __fmul_rn(xB, xB));
    }
    const uint32_t isB = dA <= dB ? 0u : 1u;
    const int fix = isB ? m : j;
    const uint32_t dofix = isB ? parB : parA;
    // A moves toward u (+1 when e < 0), B away from its first half-integer (-1 when e < 0)
    const int ef = (isB ? em : ej) < 0.0f ? 1 : -1;
    const int delta = dofix ? (isB ? -ef : ef) : 0;
    return isB | ((uint32_t)fix << 1) | ((uint32_t)(delta + 1) << 4);
}

// E8 = D8 u (D8 + 1/2), fused with bit-stripping.  Returns the coset bit c and writes the 8
// symbols (w0 .. w6, (w7 - p)/2) of the nearest point v/2 (v doubled coordinates, w = (v - c)/2);
// v itself when WANT_V.  The coset choice compares
// |u-A|^2 - |u-B|^2 = sum(|e| - 1/4) + [A fixed](1 - 2 max|e|) - [B fixed](2 min|e|) in binary32
// as D = ((S - 2) + cA) - cB, S the pairwise sum of |e|; B only when D > 0.  Within 2^-16 of a tie
// (and where a fix-up meets the 2^-31 key floor) e8_plain_choice decides instead.
//   A: w = a; if sum a is odd the coordinate with max |e| moves toward u.
//   B: w = a - [e >= 0] (w + 1/2 is the half-integer toward u); if sum w is odd the coordinate
//      with min |e| moves to its other half-integer neighbour.
// E8 decision from t = u + 1.5*2^23 and e = (t - 1.5*2^23) - u (computed by the caller)
// DEFER: instead of running the plain rule here, set `rare` and return the shortcut's point; the
// caller then redoes the block with e8_symbols (which never defers).  Kept out of the unrolled
// quantizer body, the rare branch does not split its straight-line code.
template <bool WANT_V, bool DEFER = false>
__device__ __forceinline__ uint32_t e8_from_te(const float (&tv)[8], const float (&ev)[8], int32_t (&s)[8], int32_t* v,
                                               uint32_t* rare = nullptr)
{
    int32_t a[8];
    float ae[8];
    uint32_t eb[8];
    uint32_t kmax = 0u, kmin = 0xFFFFFFFFu, tx = 0u, sx = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float t = tv[i];
        a[i] = __float_as_int(t) - __float_as_int(kMagic);
        const float e = ev[i];
        ae[i] = fabsf(e);
        eb[i] = __float_as_uint(e);
        const uint32_t key = max_key(e, i, 8);
        kmax = max(kmax, key);
        kmin = min(kmin, key ^ 0xEu);  // index bits flipped: ties go to the lowest index
        tx ^= __float_as_uint(t);      // bit 0: parity of sum a (the magic constant is even)
        sx ^= eb[i];                   // bit 31: parity of #{e < 0} (e is never -0)
    }
    const uint32_t parA = tx & 1u;
    const uint32_t parB = parA ^ (sx >> 31);  // sum w = sum a - #{e >= 0}, and 8 is even
    const float S = __fadd_rn(__fadd_rn(__fadd_rn(ae[0], ae[1]), __fadd_rn(ae[2], ae[3])),
                              __fadd_rn(__fadd_rn(ae[4], ae[5]), __fadd_rn(ae[6], ae[7])));
    const float cA = parA ? __fadd_rn(1.0f, -__fmul_rn(2.0f, key_value(kmax))) : 0.0f;
    const float cB = parB ? __fmul_rn(2.0f, key_value(kmin)) : 0.0f;
    const float D = __fadd_rn(__fadd_rn(__fadd_rn(S, -2.0f), cA), -cB);
    bool isB = D > 0.0f;
    // the coordinate to fix and its direction: A moves toward u (+1 when e < 0), B away from it
    const uint32_t kf = isB ? kmin : kmax;
    int fix = isB ? (int)((kmin >> 1) & 7u) : 7 - (int)((kmax >> 1) & 7u);
    const uint32_t dofix = isB ? parB : parA;
    int32_t delta = dofix ? ((((kf & 1u) != 0u) != isB) ? 1 : -1) : 0;
    // near a coset tie, or where a fix-up meets the 2^-31 floor of the keys: the plain rule
    const bool plain = fabsf(D) <= kTieBand || (parA && kmax < 16u) || (parB && kmin < 16u);
    if constexpr (DEFER) {
        *rare = plain ? 1u : 0u;
    } else {
        if (plain) {
            const uint32_t r = e8_plain_choice(ev[0], ev[1], ev[2], ev[3], ev[4], ev[5], ev[6], ev[7], parA, parB);
            isB = (r & 1u) != 0u;
            fix = (int)((r >> 1) & 7u);
            delta = (int32_t)(r >> 4) - 1;
        }
    }
    const uint32_t bmask = isB ? 0xFFFFFFFFu : 0u;
    int32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        w[i] = a[i] - (int32_t)((~eb[i] & bmask) >> 31);
        if (i == fix) w[i] += delta;
    }
    const int32_t p = (w[0] ^ w[1] ^ w[2] ^ w[3] ^ w[4] ^ w[5] ^ w[6]) & 1;
#pragma unroll
    for (int i = 0; i < 7; ++i) s[i] = w[i];
    s[7] = (w[7] - p) >> 1;
    const uint32_t c = isB ? 1u : 0u;
    if constexpr (WANT_V) {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 2 * w[i] + (int32_t)c;
    }
    return c;
}

template <bool WANT_V>
__device__ __forceinline__ uint32_t e8_symbols(const float (&u)[8], int32_t (&s)[8], int32_t* v)
{
    float t[8], e[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        t[i] = __fadd_rn(u[i], kMagic);
        e[i] = __fadd_rn(__fadd_rn(t[i], -kMagic), -u[i]);
    }
    return e8_from_te<WANT_V>(t, e, s, v);
}

// two E8 blocks at once, one in each lane of eight float2 pairs: the rounding arithmetic runs on
// paired binary32 operations (the same roundings as e8_symbols), the decisions per lane.  rare:
// bit 0 (lane x) / bit 1 (lane y) set where the block must be redone with e8_symbols.
template <bool WANT_V>
__device__ __forceinline__ void e8_pair_symbols(const float2 (&p)[8], int32_t (&sx)[8], int32_t (&sy)[8],
                                                uint32_t& cx, uint32_t& cy, int32_t* vx, int32_t* vy, uint32_t& rare)
{
    float tx[8], ty[8], ex[8], ey[8];
    const float2 m2 = make_float2(kMagic, kMagic);
    const float2 nm2 = make_float2(-kMagic, -kMagic);
    const float2 neg1 = make_float2(-1.0f, -1.0f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 t = __fadd2_rn(p[i], m2);
        const float2 r = __fadd2_rn(t, nm2);
        const float2 e = __ffma2_rn(p[i], neg1, r);  // r - u, exact product
        tx[i] = t.x; ty[i] = t.y;
        ex[i] = e.x; ey[i] = e.y;
    }
    uint32_t rx, ry;
    cx = e8_from_te<WANT_V, true>(tx, ex, sx, vx, &rx);
    cy = e8_from_te<WANT_V, true>(ty, ey, sy, vy, &ry);
    rare = rx | (ry << 1);
}

// A2 with minimum distance 1 in (P, Q) = (2 u0, u1 K): the even point when |eP| + 3|eQ| <= 1, which is
// |even|^2 <= |odd|^2 up to a factor of 4; near the tie the two distances themselves decide.
__device__ __forceinline__ void q_a2_pq(const float P, const float Q, int32_t (&v)[2])
{
    const float hP = __fmul_rn(P, 0.5f), hQ = __fmul_rn(Q, 0.5f);
    int32_t aP, aQ;
    const float rP = rint_magic(hP, aP), rQ = rint_magic(hQ, aQ);
    const float eP = __fadd_rn(rP, -hP), eQ = __fadd_rn(rQ, -hQ);
    const float E = __fadd_rn(fabsf(eP), __fmul_rn(3.0f, fabsf(eQ)));
    bool even = E <= 1.0f;
    if (fabsf(__fadd_rn(E, -1.0f)) <= kTieBand) {
        // near the tie of the two cosets: both candidates' dP^2 + 3 dQ^2 in binary32
        const float oP = (float)(2 * aP + ((eP < 0.0f) ? 1 : -1)), oQ = (float)(2 * aQ + ((eQ < 0.0f) ? 1 : -1));
        const float dPe = __fadd_rn(P, -(float)(2 * aP)), dQe = __fadd_rn(Q, -(float)(2 * aQ));
        const float dPo = __fadd_rn(P, -oP), dQo = __fadd_rn(Q, -oQ);
        const float de = __fadd_rn(__fmul_rn(dPe, dPe), __fmul_rn(3.0f, __fmul_rn(dQe, dQe)));
        const float dO = __fadd_rn(__fmul_rn(dPo, dPo), __fmul_rn(3.0f, __fmul_rn(dQo, dQo)));
        even = de <= dO;
    }
    if (even) {
        v[0] = 2 * aP;
        v[1] = 2 * aQ;
    } else {
        v[0] = 2 * aP + ((eP < 0.0f) ? 1 : -1);
        v[1] = 2 * aQ + ((eQ < 0.0f) ? 1 : -1);
    }
}

__device__ __forceinline__ void q_a2(const float (&u)[2], int32_t (&v)[2])
{
    q_a2_pq(__fmul_rn(2.0f, u[0]), __fmul_rn(u[1], kA2K), v);
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

// nearest point of one block and its stripped symbols: u[d] -> symbols s[d] (+ E8 coset bit);
// the integer embedding v[d] is written when WANT_V
template <int LAT, bool WANT_V>
__device__ __forceinline__ uint32_t quantize_strip(const float* u, int32_t* s, int32_t* v)
{
    if constexpr (LAT == HQ_E8) {
        float uu[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) uu[i] = u[i];
        int32_t ss[8];
        const uint32_t c = e8_symbols<WANT_V>(uu, ss, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) s[i] = ss[i];
        return c;
    } else {
        int32_t vv[Lat<LAT>::d];
        if constexpr (LAT == HQ_Z) {
            rint_magic(u[0], vv[0]);
        } else if constexpr (LAT == HQ_A2) {
            const float uu[2] = {u[0], u[1]};
            int32_t t2[2];
            q_a2(uu, t2);
            vv[0] = t2[0];
            vv[1] = t2[1];
        } else {
            const float uu[4] = {u[0], u[1], u[2], u[3]};
            int32_t t4[4];
            q_d4(uu, t4);
#pragma unroll
            for (int i = 0; i < 4; ++i) vv[i] = t4[i];
        }
        if constexpr (WANT_V) {
#pragma unroll
            for (int i = 0; i < Lat<LAT>::d; ++i) v[i] = vv[i];
        }
        return strip_block<LAT>(vv, s);
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
        const int32_t p = (s[0] ^ s[1] ^ s[2] ^ s[3] ^ s[4] ^ s[5] ^ s[6]) & 1;
#pragma unroll
        for (int i = 0; i < 7; ++i) v[i] = 2 * s[i] + (int32_t)c;
        v[7] = 2 * (2 * s[7] + p) + (int32_t)c;
    }
}

// Subtractive dither ("Subtractive Dither", Methodology step 4): U uniform on the Voronoi cell,
// in the coordinates the quantizer works in (u for Z, D4, E8; (P, Q) for A2).  Groups 2b and 2b + 1
// of four consecutive coefficients of a tile share one Philox block with counter (c_lo, c1,
// 0x80000000 | b, c_hi) under the seed's round keys rk: c = s and c1 = b H + h for KV row
// (b H + h, s); c = row and c1 = tile column for the weight-path option.  Its eight 16-bit halves
// (low half of word i first) give r = box (h + 1/2) 2^-16, the midpoints of 2^16 bins of
// [0, box) (box 1 for Z, 2 otherwise), a union of fundamental domains (2Z^d lies in D4, in E8 and
// in the (P, Q) lattice), so U = r - Q(r) is uniform on the cell up to the bins.  E8 blocks take
// one Philox block (two groups).
__device__ __forceinline__ void dither_r8(const uint32_t (&rk)[20], uint32_t c1, uint64_t c, uint32_t b, float box,
                                          float (&r)[8])
{
    const uint4 w = philox4x32_10_rk(make_uint4((uint32_t)c, c1, 0x80000000u | b, (uint32_t)(c >> 32)), rk);
    // (2h + 1) 2^-16 box: a 17-bit odd integer times a power of two, exact
    const float sc = box == 1.0f ? 7.62939453125e-06f : 1.52587890625e-05f;
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        r[2 * i] = __fmul_rn((float)(((ws[i] & 0xFFFFu) << 1) | 1u), sc);
        r[2 * i + 1] = __fmul_rn((float)(((ws[i] >> 15) & 0x1FFFEu) | 1u), sc);
    }
}

// U for the eight coefficients of groups 2b, 2b + 1 (Z: eight blocks, A2: four, D4: two)
template <int LAT>
__device__ __forceinline__ void dither_pair(const uint32_t (&rk)[20], uint32_t c1, uint64_t c, uint32_t b,
                                            float (&U)[8])
{
    static_assert(LAT != HQ_E8, "E8: dither_e8");
    float r[8];
    dither_r8(rk, c1, c, b, LAT == HQ_Z ? 1.0f : 2.0f, r);
    if constexpr (LAT == HQ_Z) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            int32_t a;
            U[i] = __fadd_rn(r[i], -rint_magic(r[i], a));
        }
    } else if constexpr (LAT == HQ_A2) {
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
            int32_t v[2];
            q_a2_pq(r[2 * bb], r[2 * bb + 1], v);
            U[2 * bb] = __fadd_rn(r[2 * bb], -(float)v[0]);
            U[2 * bb + 1] = __fadd_rn(r[2 * bb + 1], -(float)v[1]);
        }
    } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float rr[4] = {r[4 * h], r[4 * h + 1], r[4 * h + 2], r[4 * h + 3]};
            int32_t q[4];
            q_d4(rr, q);
#pragma unroll
            for (int i = 0; i < 4; ++i) U[4 * h + i] = __fadd_rn(rr[i], -(float)q[i]);
        }
    }
}

// U for the E8 block made of groups g0, g0 + 1 (g0 even; u units)
__device__ __forceinline__ void dither_e8(const uint32_t (&rk)[20], uint32_t c1, uint64_t c, uint32_t g0, float (&U)[8])
{
    float r[8];
    dither_r8(rk, c1, c, g0 >> 1, 2.0f, r);
    int32_t s[8], v[8];
    e8_symbols<true>(r, s, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) U[i] = __fadd_rn(r[i], -__fmul_rn(0.5f, (float)v[i]));
}

}  // namespace hq
