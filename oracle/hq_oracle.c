/*
 * hq_oracle.c -- plain, slow, single-threaded CPU oracle of the HyperQuant tile codec.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark may load this file's library.  The product (the CUDA library and its Python
 * binding) never links, imports or calls it, and the two share no code, header or table.
 *
 * Source of the method: "HyperQuant: A Rate-Distortion-Optimal Quantization Pipeline for Large
 * Language and Diffusion Models" (Domb, Sackstein, Solberg), as summarised on gist.science
 * (English "Technical Summary", section "Methodology: The HyperQuant Pipeline"):
 *   1. per-tile Randomized Hadamard Transform RHT_n(x) = H_n D x, D a random sign diagonal;
 *   2. nearest-point quantization to E8, D4, A2 or Z, mapped to an integer embedding;
 *   3. lossless bit-stripping of lattice-parity-fixed bits, then Rice coding;
 *   4. for the KV cache, subtractive dither U ~ Uniform(V(Lambda)) added before quantization
 *      and subtracted after.
 * The pages fix only this shape.  Every constant, order, tie rule and bit layout below is a
 * reading of them; each is listed with its reason in the repository's design notes.
 *
 * Arithmetic.  The encode chain (RMS, scale, sign flip, FWHT, normalisation, lattice decision)
 * runs in IEEE binary32 with round-to-nearest-even, no fused multiply-add (built with
 * -ffp-contract=off), correctly rounded division and square root.  It decides integer codes, so
 * it uses the same precision the device kernels use.  Decode (reconstruction) runs in binary64.
 *
 * Parity pins (all in tests/, marked "not gpu"):
 *   philox           : curand's host Philox4x32-10 generator (a library run);
 *   bf16 rounding    : torch's float32 -> bfloat16 conversion;
 *   fwht             : scipy's Sylvester Hadamard matrix product, orthogonality, exact inverse;
 *   rms              : numpy float64 RMS within binary32 rounding;
 *   lattice decoders : brute-force search over neighbouring lattice points, textbook normalised
 *                      second moments (Conway & Sloane, SPLAG, Table 2.3);
 *   rice / layout    : round trip, length formula, sum(q) <= n;
 *   codec            : inputs built on lattice points decode exactly; dithered KV inner
 *                      products are unbiased over seeds (Appendix A claim).
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#if !defined(FLT_EVAL_METHOD) || FLT_EVAL_METHOD != 0
#error "the oracle needs binary32 evaluation without excess precision"
#endif

#define HQO_Z 0
#define HQO_A2 1
#define HQO_D4 2
#define HQO_E8 3

/* status bits: bit (1 << code), codes as documented for the library's status word */
#define HQO_ST_CAPACITY (1u << 3)
#define HQO_ST_NONFINITE (1u << 4)
#define HQO_ST_CORRUPT (1u << 5)

#define HQO_MAXN 256

/* ------------------------------------------------------------------------------------------ */
/* Philox4x32-10, from Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2,  */
/* 3" (SC'11): ten rounds of two 32x32->64 multiplies with the published multipliers, the key  */
/* bumped by the published Weyl constants between rounds.                                      */
/* ------------------------------------------------------------------------------------------ */
void hqo_philox4x32_10(const uint32_t ctr[4], uint32_t key0, uint32_t key1, uint32_t out[4])
{
    uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint32_t k0 = key0, k1 = key1;
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)x0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)x2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t y0 = hi1 ^ x1 ^ k0;
        uint32_t y1 = lo1;
        uint32_t y2 = hi0 ^ x3 ^ k1;
        uint32_t y3 = lo0;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* Sign of the random diagonal D for transformed-axis index J (global column for weights, head
 * dimension index for KV).  Reading: D depends only on the seed and J, so one diagonal serves
 * every row / token and (R w).(R x) = w.x holds across rows.  One Philox block covers 128 J. */
int hqo_sign_negative(uint64_t seed, int64_t J)
{
    uint32_t ctr[4] = {(uint32_t)((uint64_t)J >> 7), 0u, 0u, 0u};
    uint32_t w[4];
    hqo_philox4x32_10(ctr, (uint32_t)seed, (uint32_t)(seed >> 32), w);
    return (int)((w[(J & 127) >> 5] >> (J & 31)) & 1u);
}

/* ------------------------------------------------------------------------------------------ */
/* bfloat16 helpers                                                                            */
/* ------------------------------------------------------------------------------------------ */
float hqo_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* round to nearest, ties to even; NaN stays NaN */
uint16_t hqo_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* c_n = 1/sqrt(n) in binary32: exact for n = 64 and 256, RN(2^-3.5) for n = 128 */
static float inv_sqrt_n(int n)
{
    if (n == 64) return 0.125f;
    if (n == 128) return f32_from_bits(0x3DB504F3u);
    return 0.0625f;
}

/* ------------------------------------------------------------------------------------------ */
/* Per-tile RMS: q_i = x_i * x_i, summed by the ascending pairwise tree (h = 1, 2, ..., n/2;   */
/* q[i] += q[i+h] for i = 0 mod 2h), s = sqrt(q[0] * (1/n)).  per-tile scaling (Methodology    */
/* step 2), RMS statistic as the workload description fixes it.                                */
/* ------------------------------------------------------------------------------------------ */
float hqo_rms(const float* x, int n)
{
    float q[HQO_MAXN];
    for (int i = 0; i < n; ++i) q[i] = x[i] * x[i];
    for (int h = 1; h < n; h *= 2)
        for (int i = 0; i < n; i += 2 * h) q[i] = q[i] + q[i + h];
    float ms = q[0] * (1.0f / (float)n);
    return sqrtf(ms);
}

/* ------------------------------------------------------------------------------------------ */
/* Fast Walsh-Hadamard transform, Sylvester (natural) order, unnormalised, butterflies in      */
/* descending stride order h = n/2, n/4, ..., 1.  (Methodology step 1: H_n.)                   */
/* ------------------------------------------------------------------------------------------ */
void hqo_fwht_f32(float* x, int n)
{
    for (int h = n / 2; h >= 1; h /= 2)
        for (int i = 0; i < n; ++i)
            if ((i & h) == 0) {
                float a = x[i], b = x[i + h];
                x[i] = a + b;
                x[i + h] = a - b;
            }
}

void hqo_fwht_f64(double* x, int n)
{
    for (int h = n / 2; h >= 1; h /= 2)
        for (int i = 0; i < n; ++i)
            if ((i & h) == 0) {
                double a = x[i], b = x[i + h];
                x[i] = a + b;
                x[i + h] = a - b;
            }
}

/* ------------------------------------------------------------------------------------------ */
/* Lattice nearest point (Methodology step 2).  Closest-point rules after Conway & Sloane,     */
/* "Fast quantizing and decoding algorithms for lattice quantizers and codes" (IEEE T-IT 1982).*/
/* Shared pieces:                                                                              */
/*   a = rint(u) (ties to even), e = a - u (exact in binary32, and never -0);                  */
/*   "toward u" for a coordinate is +1 when e < 0, else -1 (so an exact integer u, e = 0,      */
/*   re-rounds downward);                                                                      */
/*   argmax / argmin of |e| compare the exact binary32 values and break ties to the lowest     */
/*   index.                                                                                    */
/* Where two cosets compete (E8, A2) both candidate points are formed and their squared        */
/* Euclidean distances to the input are computed plainly in binary32 (coordinate differences,  */
/* squares and a sum in coordinate order, each rounded once); the first coset wins ties.       */
/* ------------------------------------------------------------------------------------------ */
static int toward(float e) { return (e < 0.0f) ? 1 : -1; }

static int argmax_abs(const float* e, int d)
{
    int j = 0;
    float best = fabsf(e[0]);
    for (int i = 1; i < d; ++i) {
        float v = fabsf(e[i]);
        if (v > best) { best = v; j = i; }
    }
    return j;
}

static int argmin_abs(const float* e, int d)
{
    int j = 0;
    float best = fabsf(e[0]);
    for (int i = 1; i < d; ++i) {
        float v = fabsf(e[i]);
        if (v < best) { best = v; j = i; }
    }
    return j;
}

/* Z: the integer nearest to u */
static void q_z(const float* u, int32_t* v) { v[0] = (int32_t)rintf(u[0]); }

/* D4 = { v in Z^4 : sum v even }.  Round each coordinate; if the sum is odd, move the
 * coordinate with the largest rounding error one step toward u. */
void hqo_q_d4(const float* u, int32_t* v)
{
    float e[4];
    int32_t a[4];
    int sum = 0;
    for (int i = 0; i < 4; ++i) {
        float r = rintf(u[i]);
        e[i] = r - u[i];
        a[i] = (int32_t)r;
        sum += a[i];
    }
    if (sum & 1) {
        int j = argmax_abs(e, 4);
        a[j] += toward(e[j]);
    }
    for (int i = 0; i < 4; ++i) v[i] = a[i];
}

/* squared distance from z to the integer point p, binary32, summed in coordinate order */
static float dist2_int(const float* z, const int32_t* p, int d)
{
    float s = 0.0f;
    for (int i = 0; i < d; ++i) {
        float t = z[i] - (float)p[i];
        s = s + t * t;
    }
    return s;
}

/* E8 = D8 u (D8 + 1/2), min norm sqrt(2), in doubled coordinates z = 2u, where its points are
 * the integer vectors with all coordinates of one parity and sum = 0 mod 4.
 *   Coset A (2 D8, even integers): p_i = 2 rint(u_i); if sum p = 2 mod 4, the coordinate with
 *     the largest |e| moves by 2 toward z.
 *   Coset B (2 D8 + 1, odd integers): p_i = the odd integer nearest z_i, 2 a_i + toward(e_i);
 *     if sum p = 2 mod 4, the coordinate farthest from its odd integer -- the one with the
 *     smallest |e|, since |z_i - p_i| = 1 - 2|e_i| -- moves by 2 to its other odd neighbour.
 *   The output is the candidate with the smaller squared distance to z (A on ties). */
void hqo_q_e8(const float* u, int32_t* v)
{
    float z[8], e[8];
    int32_t a[8], pA[8], pB[8];
    int32_t sumA = 0, sumB = 0;
    for (int i = 0; i < 8; ++i) {
        float r = rintf(u[i]);
        z[i] = 2.0f * u[i];
        e[i] = r - u[i];
        a[i] = (int32_t)r;
    }
    for (int i = 0; i < 8; ++i) {
        pA[i] = 2 * a[i];
        sumA += pA[i];
        pB[i] = 2 * a[i] + toward(e[i]);
        sumB += pB[i];
    }
    if ((sumA & 3) == 2) {
        int j = argmax_abs(e, 8);
        pA[j] += 2 * toward(e[j]);
    }
    if ((sumB & 3) == 2) {
        int m = argmin_abs(e, 8);
        pB[m] -= 2 * toward(e[m]);
    }
    float dA = dist2_int(z, pA, 8);
    float dB = dist2_int(z, pB, 8);
    const int32_t* p = (dA <= dB) ? pA : pB;
    for (int i = 0; i < 8; ++i) v[i] = p[i];
}

/* A2, minimum distance 1: points (P/2, Q*sqrt(3)/2) with P = Q mod 2.  Work in (P, Q) =
 * (2 u0, u1 * K), K = RN(2/sqrt 3), where A2 is the union of the even coset 2Z x 2Z and the
 * odd coset (2Z+1) x (2Z+1) and squared distances weigh dQ three times.  Per coordinate X the
 * nearest even integer is 2 rint(X/2) and the nearest odd one 2 rint(X/2) + toward(rint(X/2) -
 * X/2).  The output is the candidate with the smaller dP^2 + 3 dQ^2 (the even one on ties). */
static const float A2_K = 1.15470053837925153f; /* RN(2/sqrt(3)) */

static float a2_dist2(float P, float Q, const int32_t* p)
{
    float dP = P - (float)p[0], dQ = Q - (float)p[1];
    return dP * dP + 3.0f * (dQ * dQ);
}

/* A2 nearest point given (P, Q) directly (the dither is added in these coordinates). */
void hqo_q_a2_pq(float P, float Q, int32_t* v)
{
    float hP = P * 0.5f, hQ = Q * 0.5f;
    float rP = rintf(hP), rQ = rintf(hQ);
    int32_t aP = (int32_t)rP, aQ = (int32_t)rQ;
    int32_t even[2] = {2 * aP, 2 * aQ};
    int32_t odd[2] = {2 * aP + toward(rP - hP), 2 * aQ + toward(rQ - hQ)};
    if (a2_dist2(P, Q, even) <= a2_dist2(P, Q, odd)) {
        v[0] = even[0];
        v[1] = even[1];
    } else {
        v[0] = odd[0];
        v[1] = odd[1];
    }
}

void hqo_q_a2(const float* u, int32_t* v) { hqo_q_a2_pq(2.0f * u[0], u[1] * A2_K, v); }

static int lattice_dim(int lattice)
{
    switch (lattice) {
    case HQO_Z: return 1;
    case HQO_A2: return 2;
    case HQO_D4: return 4;
    default: return 8;
    }
}

static void quantize_block(int lattice, const float* u, int32_t* v)
{
    switch (lattice) {
    case HQO_Z: q_z(u, v); break;
    case HQO_A2: hqo_q_a2(u, v); break;
    case HQO_D4: hqo_q_d4(u, v); break;
    default: hqo_q_e8(u, v); break;
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Bit-stripping (Methodology step 3): drop the bits the lattice's parity checks fix.          */
/*   E8 : c = v0 & 1 (coset bit, sent raw); w = (v - c)/2 in D8; p = (w0+..+w6) & 1;          */
/*        symbols w0..w6, (w7 - p)/2.                                                          */
/*   D4 : p = (v0+v1+v2) & 1; symbols v0, v1, v2, (v3 - p)/2.                                  */
/*   A2 : symbols P, (Q - (P & 1))/2.                                                          */
/*   Z  : the symbol is v.                                                                     */
/* Every lattice yields one symbol per coordinate.                                             */
/* ------------------------------------------------------------------------------------------ */
static void strip_block(int lattice, const int32_t* v, int32_t* sym, int* coset)
{
    *coset = 0;
    if (lattice == HQO_Z) {
        sym[0] = v[0];
    } else if (lattice == HQO_A2) {
        sym[0] = v[0];
        sym[1] = (v[1] - (v[0] & 1)) >> 1;
    } else if (lattice == HQO_D4) {
        int p = (v[0] + v[1] + v[2]) & 1;
        sym[0] = v[0]; sym[1] = v[1]; sym[2] = v[2];
        sym[3] = (v[3] - p) >> 1;
    } else {
        int c = v[0] & 1;
        int32_t w[8];
        for (int i = 0; i < 8; ++i) w[i] = (v[i] - c) >> 1;
        int p = (w[0] + w[1] + w[2] + w[3] + w[4] + w[5] + w[6]) & 1;
        for (int i = 0; i < 7; ++i) sym[i] = w[i];
        sym[7] = (w[7] - p) >> 1;
        *coset = c;
    }
}

static void unstrip_block(int lattice, const int32_t* sym, int coset, int32_t* v)
{
    if (lattice == HQO_Z) {
        v[0] = sym[0];
    } else if (lattice == HQO_A2) {
        v[0] = sym[0];
        v[1] = 2 * sym[1] + (sym[0] & 1);
    } else if (lattice == HQO_D4) {
        int p = (sym[0] + sym[1] + sym[2]) & 1;
        v[0] = sym[0]; v[1] = sym[1]; v[2] = sym[2];
        v[3] = 2 * sym[3] + p;
    } else {
        int p = (sym[0] + sym[1] + sym[2] + sym[3] + sym[4] + sym[5] + sym[6]) & 1;
        int32_t w[8];
        for (int i = 0; i < 7; ++i) w[i] = sym[i];
        w[7] = 2 * sym[7] + p;
        for (int i = 0; i < 8; ++i) v[i] = 2 * w[i] + coset;
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Rice coding (Methodology step 3).  zz = 2m (m >= 0) or -2m-1 (m < 0); the tile parameter   */
/* k = min{k >= 0 : sum zz < n 2^(k+1)}, capped at 15 -- k follows the mean index: k is the   */
/* smallest k with mean(zz) < 2^(k+1), the rational form of the mean-based Rice parameter that  */
/* is optimal for geometric sources (it codes Gaussian-like symbols within ~0.06 bit of their  */
/* entropy, where k = ceil(log2 mean) loses ~0.3 bit).  q = zz >> k, r = zz & (2^k - 1).  Below */
/* the cap, sum zz < n 2^(k+1) gives sum q < 2n.                                               */
/* Tile bit string.  Bit position p of a chunk lives in 32-bit word p >> 5 at bit p & 31.      */
/* A symbol's Rice code is, in reading order: q zeros, a one, then r in k bits, most           */
/* significant first.  The tile holds                                                          */
/*   [E8 only: n/8 coset bits, block b at offset b]                                            */
/*   [symbols 0 .. n/2-1, read forward (increasing position) from offset n/8 (E8) or 0]        */
/*   [symbols n-1 down to n/2, read backward (decreasing position) from the tile's last bit]   */
/* The second half is written from the tile's end so that each half can be decoded on its own */
/* knowing only the tile length L = (E8 ? n/8 : 0) + n (k + 1) + sum q, which k and sum q       */
/* (stored per tile) give; the two halves meet exactly.                                        */
/* ------------------------------------------------------------------------------------------ */
static uint32_t zigzag(int32_t m) { return m >= 0 ? (uint32_t)m * 2u : (uint32_t)(-(int64_t)m) * 2u - 1u; }
static int32_t unzigzag(uint32_t z) { return (z & 1u) ? -(int32_t)((z + 1u) >> 1) : (int32_t)(z >> 1); }

static int rice_k(uint64_t A, int n)
{
    int k = 0;
    while (k < 15 && !(A < ((uint64_t)n << (k + 1)))) ++k;
    return k;
}

typedef struct {
    uint32_t* words;
    int64_t cap_words;
    int64_t bitpos; /* absolute bit position in words[] where the next tile starts */
    int overflow;
} bitw_t;

static void set_bit(bitw_t* w, int64_t pos, int bit)
{
    int64_t wi = pos >> 5;
    if (wi >= w->cap_words) {
        w->overflow = 1;
    } else if (bit) {
        w->words[wi] |= 1u << (pos & 31);
    }
}

/* writes one Rice code at *pos, moving by step (+1 forward, -1 backward) */
static void put_code(bitw_t* w, int64_t* pos, int step, uint32_t q, uint32_t r, int k)
{
    for (uint32_t j = 0; j < q; ++j) { set_bit(w, *pos, 0); *pos += step; }
    set_bit(w, *pos, 1);
    *pos += step;
    for (int b = k - 1; b >= 0; --b) { set_bit(w, *pos, (int)((r >> b) & 1u)); *pos += step; }
}

typedef struct {
    const uint32_t* words;
    int64_t nwords;
    int bad;
} bitr_t;

static int get_bit(bitr_t* r, int64_t pos)
{
    int64_t wi = pos >> 5;
    if (pos < 0 || wi >= r->nwords) {
        r->bad = 1;
        return 0;
    }
    return (int)((r->words[wi] >> (pos & 31)) & 1u);
}

/* reads one Rice code at *pos moving by step; returns 0 on a run longer than limit */
static int get_code(bitr_t* rd, int64_t* pos, int step, int k, uint32_t limit, uint32_t* q_out, uint32_t* r_out)
{
    uint32_t q = 0;
    while (!get_bit(rd, *pos)) {
        *pos += step;
        if (rd->bad || ++q > limit) return 0;
    }
    *pos += step;
    uint32_t r = 0;
    for (int b = 0; b < k; ++b) { r = (r << 1) | (uint32_t)get_bit(rd, *pos); *pos += step; }
    *q_out = q;
    *r_out = r;
    return !rd->bad;
}

/* ------------------------------------------------------------------------------------------ */
/* Subtractive dither (Methodology step 4): U uniform on the Voronoi cell of the lattice, in   */
/* the coordinates its quantizer works in (u for Z, D4, E8; (P, Q) = (2 u0, u1 K) for A2).     */
/* Groups 2b and 2b + 1 of four consecutive coefficients of a tile share one Philox block: key  */
/* = seed, counter (c_lo, c1, 0x80000000 | b, c_hi) with c = s for the KV row (b H + h, s),     */
/* c1 = b H + h (the weight-path option uses c = row, c1 = tile column).  Its 128 bits are      */
/* eight 16-bit halves h_0 .. h_7 (h_2i the low half of word i): group 2b takes h_0 .. h_3,      */
/* group 2b + 1 h_4 .. h_7, and r = box (h + 1/2) 2^-16, the midpoints of 2^16 equal bins of      */
/* [0, box) (mean exactly box / 2): box 1 for Z, 2 for the others.  Each box is a union of      */
/* fundamental domains (Z^1; 2Z^4 in D4; 2Z^8 in E8, which holds D8; 2Z^2 in the (P, Q) lattice  */
/* P = Q mod 2), so U = r - Q(r) is uniform on the Voronoi cell up to the 2^-16 bins.  E8       */
/* blocks take groups 2b and 2b + 1, one Philox block each.                                      */
/* ------------------------------------------------------------------------------------------ */
static void dither_group(uint64_t seed, int64_t c1, int64_t c, int g, float box, float r[4])
{
    uint32_t ctr[4] = {(uint32_t)(uint64_t)c, (uint32_t)(uint64_t)c1, 0x80000000u | (uint32_t)(g >> 1),
                       (uint32_t)((uint64_t)c >> 32)};
    uint32_t w[4];
    hqo_philox4x32_10(ctr, (uint32_t)seed, (uint32_t)(seed >> 32), w);
    for (int i = 0; i < 4; ++i) {
        int j = 4 * (g & 1) + i; /* half index within the block */
        uint32_t h = (w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
        r[i] = box * ((float)(2u * h + 1u) * 7.62939453125e-06f); /* box (h + 1/2) 2^-16 = box (2h + 1) 2^-17, exact */
    }
}

/* U for all n coefficients of one tile */
void hqo_dither(int lattice, uint64_t seed, int64_t c1, int64_t c, int n, float* U)
{
    const float box = lattice == HQO_Z ? 1.0f : 2.0f;
    float r[HQO_MAXN];
    for (int g = 0; g < n / 4; ++g) dither_group(seed, c1, c, g, box, r + 4 * g);
    int32_t v[8];
    switch (lattice) {
    case HQO_Z:
        for (int i = 0; i < n; ++i) U[i] = r[i] - rintf(r[i]);
        break;
    case HQO_A2:
        for (int b = 0; b < n / 2; ++b) {
            hqo_q_a2_pq(r[2 * b], r[2 * b + 1], v);
            U[2 * b] = r[2 * b] - (float)v[0];
            U[2 * b + 1] = r[2 * b + 1] - (float)v[1];
        }
        break;
    case HQO_D4:
        for (int b = 0; b < n / 4; ++b) {
            hqo_q_d4(r + 4 * b, v);
            for (int i = 0; i < 4; ++i) U[4 * b + i] = r[4 * b + i] - (float)v[i];
        }
        break;
    default:
        for (int b = 0; b < n / 8; ++b) {
            hqo_q_e8(r + 8 * b, v);  /* twice the point */
            for (int i = 0; i < 8; ++i) U[8 * b + i] = r[8 * b + i] - 0.5f * (float)v[i];
        }
        break;
    }
}

/* the D4 dither of one block (group), kept for the pins */
void hqo_dither_d4(uint64_t seed, int64_t bh, int64_t s, int blk, float U[4])
{
    float r[4];
    dither_group(seed, bh, s, blk, 2.0f, r);
    int32_t q[4];
    hqo_q_d4(r, q);
    for (int i = 0; i < 4; ++i) U[i] = r[i] - (float)q[i];
}

/* ------------------------------------------------------------------------------------------ */
/* Tile geometry.  W[rows, cols] row-major, tile (r, jt) = W[r, jt n : (jt+1) n].  Tile index  */
/* t = jt * rows + r.  Chunk (jt, rb) holds rows [32 rb, min(32 rb + 32, rows)) of tile column */
/* jt; chunk index c = jt * RB + rb with RB = ceil(rows / 32).  Chunks start on 32-bit word    */
/* boundaries; chunk_word[c] is the word offset of chunk c, chunk_word[C] the total.          */
/* ------------------------------------------------------------------------------------------ */

/* One tile from lattice-unit coefficients u (already normalised, before dither) to codes v
 * (integer embedding).  dither: add the tile's dither (counter words c1, c) first. */
static void quantize_tile(const float* u_in, int n, int lattice, int dither, uint64_t seed, int64_t c1,
                          int64_t c, int32_t* v)
{
    int d = lattice_dim(lattice);
    float z[HQO_MAXN];
    for (int i = 0; i < n; ++i) z[i] = u_in[i];
    if (!dither) {
        for (int b = 0; b < n / d; ++b) quantize_block(lattice, z + b * d, v + b * d);
        return;
    }
    float U[HQO_MAXN];
    hqo_dither(lattice, seed, c1, c, n, U);
    if (lattice == HQO_A2) {
        for (int b = 0; b < n / 2; ++b) {
            float P = 2.0f * z[2 * b], Q = z[2 * b + 1] * A2_K;
            hqo_q_a2_pq(P + U[2 * b], Q + U[2 * b + 1], v + 2 * b);
        }
        return;
    }
    for (int i = 0; i < n; ++i) z[i] = z[i] + U[i];
    for (int b = 0; b < n / d; ++b) quantize_block(lattice, z + b * d, v + b * d);
}

/* Rice-code one tile's codes into the bit writer at w->bitpos; returns k and sum q. */
static void rice_tile(const int32_t* v, int n, int lattice, bitw_t* w, int* k_out, int* sumq_out)
{
    int d = lattice_dim(lattice);
    int32_t sym[HQO_MAXN];
    int cos[HQO_MAXN / 8];
    for (int b = 0; b < n / d; ++b) {
        int c;
        strip_block(lattice, v + b * d, sym + b * d, &c);
        if (lattice == HQO_E8) cos[b] = c;
    }
    uint64_t A = 0;
    for (int i = 0; i < n; ++i) A += zigzag(sym[i]);
    int k = rice_k(A, n);
    uint32_t q[HQO_MAXN], r[HQO_MAXN];
    int sumq = 0;
    for (int i = 0; i < n; ++i) {
        uint32_t z = zigzag(sym[i]);
        q[i] = z >> k;
        r[i] = z & ((1u << k) - 1u);
        sumq += (int)q[i];
    }
    int cosb = lattice == HQO_E8 ? n / 8 : 0;
    int64_t start = w->bitpos;
    int64_t L = cosb + (int64_t)n * (k + 1) + sumq;
    for (int b = 0; b < cosb; ++b) set_bit(w, start + b, cos[b]);
    int64_t pos = start + cosb;                 /* first half, forward */
    for (int i = 0; i < n / 2; ++i) put_code(w, &pos, +1, q[i], r[i], k);
    int64_t mid = pos;
    pos = start + L - 1;                        /* second half, backward from the last bit */
    for (int i = n - 1; i >= n / 2; --i) put_code(w, &pos, -1, q[i], r[i], k);
    if (pos != mid - 1) w->overflow = 1;        /* the halves must meet exactly */
    w->bitpos = start + L;
    *k_out = k;
    *sumq_out = sumq;
}

/* Row (b*H + h, s) of a KV tensor [B, H, S, D] flattened to rows = B*H*S. */
static void kv_row(int64_t r, int64_t S, int64_t* bh, int64_t* s)
{
    if (S <= 0) { *bh = 0; *s = r; return; }
    *bh = r / S;
    *s = r % S;
}

static int valid_common(int n, int lattice)
{
    return (n == 64 || n == 128 || n == 256) && lattice >= 0 && lattice <= 3;
}

/* kv: 0 no dither; 1 KV rows (b H + h, s) with the dither; 2 weights with the dither (option) */
static int valid_kv(int kv, int lattice) { return (kv >= 0 && kv <= 2) && lattice >= 0 && lattice <= 3; }

/* dither counter words of tile (row r of the call, tile column jt); KV rows of a call that
 * starts at token s0 of every sequence (token append) are tokens s0 + r % kv_S */
static void dither_words(int kv, int64_t r, int64_t kv_S, int64_t kv_s0, int64_t jt, int64_t* c1, int64_t* c)
{
    if (kv == 1) {
        kv_row(r, kv_S, c1, c);
        *c += kv_s0;
    } else {
        *c1 = jt;
        *c = r;
    }
}

/*
 * Full encode.
 *   x       : [rows, cols] bf16 (dtype 0) or fp32 (dtype 1), row-major
 *   beta    : step (lattice units per normalised coefficient), > 0
 *   kv      : 1 = KV path (dither of row (b H + h, s)), kv_S = S of the [B,H,S,D] layout
 *             (rows = B*H*S); 2 = weights with the dither of tile (row, tile column); 0 none
 *   outputs : scale[T] (bf16 bits of the per-tile RMS), meta[T] = k | (sum q << 4),
 *             chunk_word[C+1], bits[cap_words]; optional v_out[T*n] (integer codes) and
 *             u_out[T*n] (normalised coefficients before dither)
 *   row0    : KV only: global row of x's first row (a slice of a larger KV tensor)
 * Returns a bitmask of status bits (0 = ok).
 */
uint32_t hqo_encode(const void* x, int dtype, int64_t rows, int64_t cols, int n, int lattice, float beta,
                    uint64_t seed, int kv, int64_t kv_S, uint16_t* scale, uint16_t* meta,
                    uint32_t* chunk_word, uint32_t* bits, int64_t cap_words, int32_t* v_out,
                    float* u_out, int64_t row0, int64_t kv_s0)
{
    if (!valid_common(n, lattice) || !valid_kv(kv, lattice) || rows <= 0 || cols <= 0 || cols % n) return 1u << 1;
    uint32_t status = 0;
    const int64_t NT = cols / n, RB = (rows + 31) / 32;
    const float cn = inv_sqrt_n(n);
    memset(bits, 0, (size_t)cap_words * 4);
    bitw_t w = {bits, cap_words, 0, 0};
    int64_t c = 0;
    for (int64_t jt = 0; jt < NT; ++jt) {
        for (int64_t rb = 0; rb < RB; ++rb, ++c) {
            chunk_word[c] = (uint32_t)(w.bitpos >> 5);
            int64_t r_end = (rb + 1) * 32 < rows ? (rb + 1) * 32 : rows;
            for (int64_t r = rb * 32; r < r_end; ++r) {
                int64_t t = jt * rows + r;
                float xt[HQO_MAXN], u[HQO_MAXN];
                int finite = 1;
                for (int j = 0; j < n; ++j) {
                    int64_t idx = r * cols + jt * n + j;
                    xt[j] = dtype == 0 ? hqo_bf16_to_f32(((const uint16_t*)x)[idx]) : ((const float*)x)[idx];
                    if (!isfinite(xt[j])) finite = 0;
                }
                float s = finite ? hqo_rms(xt, n) : 0.0f;
                uint16_t sh = hqo_f32_to_bf16(s);
                float shf = hqo_bf16_to_f32(sh);
                if (!finite || !isfinite(shf)) {
                    status |= HQO_ST_NONFINITE;
                    sh = 0;
                    shf = 0.0f;
                } else if (shf < 1.2621774483536189e-29f /* 2^-96 */) {
                    sh = 0;
                    shf = 0.0f;
                }
                if (shf == 0.0f) {
                    for (int j = 0; j < n; ++j) u[j] = 0.0f;
                } else {
                    for (int j = 0; j < n; ++j)
                        if (hqo_sign_negative(seed, jt * n + j)) xt[j] = -xt[j];
                    hqo_fwht_f32(xt, n);
                    float tden = shf * beta;
                    float rinv = 1.0f / tden;
                    float g = cn * rinv;
                    for (int j = 0; j < n; ++j) u[j] = xt[j] * g;
                }
                int64_t c1 = 0, cw = 0;
                if (kv) dither_words(kv, row0 + r, kv_S, kv_s0, jt, &c1, &cw);
                int32_t v[HQO_MAXN];
                quantize_tile(u, n, lattice, kv != 0, seed, c1, cw, v);
                int k, sumq;
                rice_tile(v, n, lattice, &w, &k, &sumq);
                scale[t] = sh;
                meta[t] = (uint16_t)(k | (sumq << 4));
                if (v_out) memcpy(v_out + t * n, v, sizeof(int32_t) * (size_t)n);
                if (u_out) memcpy(u_out + t * n, u, sizeof(float) * (size_t)n);
            }
            w.bitpos = (w.bitpos + 31) & ~(int64_t)31; /* chunk ends on a word boundary */
        }
    }
    chunk_word[c] = (uint32_t)(w.bitpos >> 5);
    if (w.overflow) status |= HQO_ST_CAPACITY;
    return status;
}

/*
 * Quantize caller-given normalised coefficients u[tiles, n] (lattice units): lattice + strip +
 * Rice + chunk layout with rows = tiles and one tile column.  kv = 1: the dither of KV row
 * (t / kv_S, t % kv_S) is added first; kv = 2: the dither of tile (t, 0).  Outputs as for
 * hqo_encode (no scale).
 */
static uint32_t quantize_rows(const float* u, int64_t tiles, int n, int lattice, int kv, int64_t kv_S,
                              int64_t row0, int64_t kv_s0, uint64_t seed, int32_t* v_out, uint16_t* meta,
                              uint32_t* chunk_word, uint32_t* bits, int64_t cap_words);

uint32_t hqo_quantize_coeffs(const float* u, int64_t tiles, int n, int lattice, int kv, int64_t kv_S,
                             uint64_t seed, int32_t* v_out, uint16_t* meta, uint32_t* chunk_word,
                             uint32_t* bits, int64_t cap_words)
{
    if (!valid_common(n, lattice) || !valid_kv(kv, lattice) || tiles <= 0) return 1u << 1;
    return quantize_rows(u, tiles, n, lattice, kv, kv_S, 0, 0, seed, v_out, meta, chunk_word, bits, cap_words);
}

/* rows of normalised coefficients (one tile each, chunks of 32 rows) -> codes and bitstream; the
 * dither words of row t are those of row row0 + t of a call starting at token kv_s0 */
static uint32_t quantize_rows(const float* u, int64_t tiles, int n, int lattice, int kv, int64_t kv_S,
                              int64_t row0, int64_t kv_s0, uint64_t seed, int32_t* v_out, uint16_t* meta,
                              uint32_t* chunk_word, uint32_t* bits, int64_t cap_words)
{
    memset(bits, 0, (size_t)cap_words * 4);
    bitw_t w = {bits, cap_words, 0, 0};
    int64_t RB = (tiles + 31) / 32;
    for (int64_t c = 0; c < RB; ++c) {
        chunk_word[c] = (uint32_t)(w.bitpos >> 5);
        int64_t t_end = (c + 1) * 32 < tiles ? (c + 1) * 32 : tiles;
        for (int64_t t = c * 32; t < t_end; ++t) {
            int64_t c1 = 0, cw = 0;
            if (kv) dither_words(kv, row0 + t, kv_S, kv_s0, 0, &c1, &cw);
            int32_t v[HQO_MAXN];
            quantize_tile(u + t * n, n, lattice, kv != 0, seed, c1, cw, v);
            int k, sumq;
            rice_tile(v, n, lattice, &w, &k, &sumq);
            meta[t] = (uint16_t)(k | (sumq << 4));
            if (v_out) memcpy(v_out + t * n, v, sizeof(int32_t) * (size_t)n);
        }
        w.bitpos = (w.bitpos + 31) & ~(int64_t)31;
    }
    chunk_word[RB] = (uint32_t)(w.bitpos >> 5);
    return w.overflow ? HQO_ST_CAPACITY : 0u;
}

/* Parse one tile starting at bit `start` back to integer codes, using k and sum q from meta:
 * the first half forward from the start, the second half backward from start + L - 1.  The
 * halves must meet exactly and sum q must agree.  Returns the tile length, or -1. */
static int64_t parse_tile(bitr_t* rd, int64_t start, int n, int lattice, uint16_t meta, int32_t* v)
{
    int d = lattice_dim(lattice);
    int k = meta & 15, sumq_meta = meta >> 4;
    int cosb = lattice == HQO_E8 ? n / 8 : 0;
    int64_t L = cosb + (int64_t)n * (k + 1) + sumq_meta;
    int cos[HQO_MAXN / 8];
    for (int b = 0; b < cosb; ++b) cos[b] = get_bit(rd, start + b);
    int32_t sym[HQO_MAXN];
    uint32_t q, r;
    int sumq = 0;
    int64_t pos = start + cosb;
    for (int i = 0; i < n / 2; ++i) {
        if (!get_code(rd, &pos, +1, k, (uint32_t)sumq_meta, &q, &r)) return -1;
        sumq += (int)q;
        sym[i] = unzigzag((q << k) | r);
    }
    int64_t mid = pos;
    pos = start + L - 1;
    for (int i = n - 1; i >= n / 2; --i) {
        if (!get_code(rd, &pos, -1, k, (uint32_t)sumq_meta, &q, &r)) return -1;
        sumq += (int)q;
        sym[i] = unzigzag((q << k) | r);
    }
    if (rd->bad || sumq != sumq_meta || pos != mid - 1) return -1;
    for (int b = 0; b < n / d; ++b) unstrip_block(lattice, sym + b * d, lattice == HQO_E8 ? cos[b] : 0, v + b * d);
    return L;
}

/* Parse the chunked stream to codes; tiles laid out as in hqo_encode.  Returns status bits. */
uint32_t hqo_parse(const uint16_t* meta, const uint32_t* chunk_word, const uint32_t* bits, int64_t rows,
                   int64_t cols, int n, int lattice, int32_t* v_out)
{
    if (!valid_common(n, lattice) || rows <= 0 || cols % n) return 1u << 1;
    const int64_t NT = cols / n, RB = (rows + 31) / 32;
    const int64_t nwords = chunk_word[NT * RB];
    uint32_t status = 0;
    int64_t c = 0;
    bitr_t rd = {bits, nwords, 0};
    for (int64_t jt = 0; jt < NT; ++jt)
        for (int64_t rb = 0; rb < RB; ++rb, ++c) {
            int64_t pos = (int64_t)chunk_word[c] * 32;
            int64_t r_end = (rb + 1) * 32 < rows ? (rb + 1) * 32 : rows;
            for (int64_t r = rb * 32; r < r_end; ++r) {
                int64_t t = jt * rows + r;
                rd.bad = 0;
                int64_t L = parse_tile(&rd, pos, n, lattice, meta[t], v_out + t * n);
                if (L < 0) {
                    status |= HQO_ST_CORRUPT;
                    memset(v_out + t * n, 0, sizeof(int32_t) * (size_t)n);
                    int k = meta[t] & 15;
                    L = (lattice == HQO_E8 ? n / 8 : 0) + (int64_t)n * (k + 1) + (meta[t] >> 4);
                }
                pos += L;
            }
            if (((pos + 31) >> 5) != (int64_t)chunk_word[c + 1]) status |= HQO_ST_CORRUPT;
        }
    return status;
}

/*
 * Reconstruct one tile (binary64) from its integer codes: lattice point p (u units) from the
 * codes, minus the dither when there is one, then x_hat = D H_n p * (s_hat * beta * c_n).
 *   E8: p = v / 2;  D4, Z: p = v;  A2: p = (P/2, Q sqrt(3)/2), the dither taken off P and Q.
 * H_n H_n = n I and u = (H D x) c_n / (s_hat beta) give x = D H u (s_hat beta) c_n.
 */
static void reconstruct_tile(const int32_t* v, int n, int lattice, int dither, uint64_t seed, int64_t c1,
                             int64_t c, uint16_t sh, float beta, int64_t col0, double* out)
{
    double p[HQO_MAXN];
    float U[HQO_MAXN];
    if (dither) hqo_dither(lattice, seed, c1, c, n, U);
    for (int i = 0; i < n; ++i) {
        double Ui = dither ? (double)U[i] : 0.0;
        if (lattice == HQO_E8) p[i] = 0.5 * (double)v[i] - Ui;
        else if (lattice == HQO_A2) p[i] = (i & 1) ? ((double)v[i] - Ui) * (sqrt(3.0) / 2.0) : 0.5 * ((double)v[i] - Ui);
        else p[i] = (double)v[i] - Ui;
    }
    hqo_fwht_f64(p, n);
    double h = (double)hqo_bf16_to_f32(sh) * (double)beta / sqrt((double)n);
    for (int j = 0; j < n; ++j) {
        double val = p[j] * h;
        out[j] = hqo_sign_negative(seed, col0 + j) ? -val : val;
    }
}

/* Full decode to binary64 out[rows, cols].  Returns status bits. */
uint32_t hqo_decode(const uint16_t* scale, const uint16_t* meta, const uint32_t* chunk_word, const uint32_t* bits,
                    int64_t rows, int64_t cols, int n, int lattice, float beta, uint64_t seed, int kv,
                    int64_t kv_S, double* out, int64_t row0, int64_t kv_s0)
{
    if (!valid_common(n, lattice) || !valid_kv(kv, lattice) || rows <= 0 || cols % n) return 1u << 1;
    const int64_t NT = cols / n;
    int32_t* v = (int32_t*)malloc(sizeof(int32_t) * (size_t)(rows * cols));
    if (!v) return 1u << 1;
    uint32_t status = hqo_parse(meta, chunk_word, bits, rows, cols, n, lattice, v);
    for (int64_t jt = 0; jt < NT; ++jt)
        for (int64_t r = 0; r < rows; ++r) {
            int64_t t = jt * rows + r;
            int64_t c1 = 0, cw = 0;
            if (kv) dither_words(kv, row0 + r, kv_S, kv_s0, jt, &c1, &cw);
            double tile[HQO_MAXN];
            reconstruct_tile(v + t * n, n, lattice, kv != 0, seed, c1, cw, scale[t], beta, jt * n, tile);
            memcpy(out + r * cols + jt * n, tile, sizeof(double) * (size_t)n);
        }
    free(v);
    return status;
}

/* Small helpers exposed for the pins. */
void hqo_quantize_block(int lattice, const float* u, int32_t* v) { quantize_block(lattice, u, v); }

/* m consecutive blocks of d = dim(lattice) coordinates each */
void hqo_quantize_blocks(int lattice, const float* u, int64_t m, int32_t* v)
{
    int d = lattice_dim(lattice);
    for (int64_t b = 0; b < m; ++b) quantize_block(lattice, u + b * d, v + b * d);
}

void hqo_strip_block(int lattice, const int32_t* v, int32_t* sym, int* coset) { strip_block(lattice, v, sym, coset); }

void hqo_unstrip_block(int lattice, const int32_t* sym, int coset, int32_t* v) { unstrip_block(lattice, sym, coset, v); }

/* Rice-code a tile of integer codes into words[] (no chunk padding); returns bit length. */
int64_t hqo_rice_tile(const int32_t* v, int n, int lattice, uint32_t* words, int64_t cap_words, int* k, int* sumq)
{
    memset(words, 0, (size_t)cap_words * 4);
    bitw_t w = {words, cap_words, 0, 0};
    rice_tile(v, n, lattice, &w, k, sumq);
    return w.overflow ? -1 : w.bitpos;
}

int hqo_parse_tile(const uint32_t* words, int64_t nwords, int n, int lattice, uint16_t meta, int32_t* v, int64_t* bitlen)
{
    bitr_t rd = {words, nwords, 0};
    int64_t L = parse_tile(&rd, 0, n, lattice, meta, v);
    *bitlen = L;
    return L >= 0;
}

/* ------------------------------------------------------------------------------------------ */
/* Decode-fused int8 GEMM (a next step of the method's tensor-core integration: the abstract's */
/* 8-bit MMA paths, "int8 beats fp8 on the post-RHT lattice output").  The weight's integer     */
/* codes v (RHT domain) multiply int8 activations that went through the same RHT:              */
/*   (W x)_r = sum_t h_{r,t} c_L sum_{j in t} v_{r,j} (H D x)_j / n    (H H = n I),             */
/* so with a = int8 (H D x) and a per-row activation scale sa_m:                               */
/*   Y[m, r] = sa_m * sum_t g_{r,t} S_{m,r,t},  S = sum_{j in t} a_{m,j} v_{r,j}  (exact int),  */
/*   g_{r,t} = ((s_hat beta) c_n) c_L,  c_L = 1/2 for E8 (doubled codes), 1 for Z and D4.       */
/* The group sums are exact; the scales are applied in binary32 as acc = fma(S, g, acc) over   */
/* t ascending from acc = 0, then y = acc * sa_m.                                              */
/* ------------------------------------------------------------------------------------------ */

/* group scale of one tile, binary32 as written above */
float hqo_group_scale(uint16_t sh, float beta, int n, int lattice)
{
    float cn = inv_sqrt_n(n);
    float h = (hqo_bf16_to_f32(sh) * beta) * cn;
    return lattice == HQO_E8 ? h * 0.5f : h;
}

/* codes of a weight code -> v8[rows, cols] (int8, tile (r, jt) at columns jt n ..) and
 * g[cols / n, rows]; tiles with a code outside [-127, 127] are written as zeros and flagged
 * (status bit 6, range).  Only Z, D4 and E8 without dither. */
uint32_t hqo_decode_int8(const uint16_t* scale, const uint16_t* meta, const uint32_t* chunk_word, const uint32_t* bits,
                         int64_t rows, int64_t cols, int n, int lattice, float beta, int8_t* v8, float* g)
{
    if (!valid_common(n, lattice) || lattice == HQO_A2 || rows <= 0 || cols % n) return 1u << 1;
    const int64_t NT = cols / n;
    int32_t* v = (int32_t*)malloc(sizeof(int32_t) * (size_t)(rows * cols));
    if (!v) return 1u << 1;
    uint32_t status = hqo_parse(meta, chunk_word, bits, rows, cols, n, lattice, v);
    for (int64_t jt = 0; jt < NT; ++jt)
        for (int64_t r = 0; r < rows; ++r) {
            int64_t t = jt * rows + r;
            int ok = 1;
            for (int i = 0; i < n; ++i)
                if (v[t * n + i] < -127 || v[t * n + i] > 127) ok = 0;
            if (!ok) status |= 1u << 6;
            for (int i = 0; i < n; ++i) v8[r * cols + jt * n + i] = ok ? (int8_t)v[t * n + i] : 0;
            g[jt * rows + r] = hqo_group_scale(scale[t], beta, n, lattice);
        }
    free(v);
    return status;
}

/* one output of the grouped GEMM: A[M, K], V[N, K] int8 row-major, g[K / n, N], sa[M] */
float hqo_gemm_one(const int8_t* A, const float* sa, const int8_t* V, const float* g, int64_t N, int64_t K, int n,
                   int64_t m, int64_t r)
{
    float acc = 0.0f;
    for (int64_t t = 0; t < K / n; ++t) {
        int64_t S = 0;
        for (int j = 0; j < n; ++j) S += (int64_t)A[m * K + t * n + j] * (int64_t)V[r * K + t * n + j];
        acc = fmaf((float)S, g[t * N + r], acc);
    }
    return acc * sa[m];
}

void hqo_gemm_grouped(const int8_t* A, const float* sa, int64_t M, const int8_t* V, const float* g, int64_t N,
                      int64_t K, int n, float* Y)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t r = 0; r < N; ++r) Y[m * N + r] = hqo_gemm_one(A, sa, V, g, N, K, n, m, r);
}

/* sampled outputs Y[idx_m[i], idx_r[i]] */
void hqo_gemm_grouped_sample(const int8_t* A, const float* sa, const int8_t* V, const float* g, int64_t N, int64_t K,
                             int n, const int64_t* idx_m, const int64_t* idx_r, int64_t count, float* out)
{
    for (int64_t i = 0; i < count; ++i) out[i] = hqo_gemm_one(A, sa, V, g, N, K, n, idx_m[i], idx_r[i]);
}


/* ------------------------------------------------------------------------------------------ */
/* Dense-rotation KV variant.  Methodology step 4 ("Bias Correction for KV Cache") allows the     */
/* per-layer rotation of the KV path to be either the sign diagonal or a dense random          */
/* orthogonal matrix drawn from the Haar measure (the QJL-style rotation, credited in Key       */
/* Contributions with the gain at 1.7-2.5 bps).  The caller passes Q (n x n, row-major,         */
/* y = Q x).  Reading: the RMS scale, lattice, dither, stripping and Rice coding are the        */
/* codec's; there is no sign diagonal (Q is random already) and no c_n (Q is orthonormal).      */
/* Binary32 forward: y_j = fma chain over i = 0 .. n-1 of Q[j][i] x_i from 0, then             */
/* u_j = y_j * (1 / (s_hat beta)).  Zero and non-finite tiles as the codec.                    */
/* ------------------------------------------------------------------------------------------ */
uint32_t hqo_rotate_normalize(const void* x, int dtype, int64_t rows, int n, const float* Q, float beta,
                              float* u_out, uint16_t* scale_out)
{
    if (!(n == 64 || n == 128) || rows <= 0) return 1u << 1;
    uint32_t status = 0;
    for (int64_t r = 0; r < rows; ++r) {
        float xt[HQO_MAXN];
        int finite = 1;
        for (int i = 0; i < n; ++i) {
            xt[i] = dtype == 0 ? hqo_bf16_to_f32(((const uint16_t*)x)[r * n + i]) : ((const float*)x)[r * n + i];
            if (!isfinite(xt[i])) finite = 0;
        }
        float s = finite ? hqo_rms(xt, n) : 0.0f;
        uint16_t sh = hqo_f32_to_bf16(s);
        float shf = hqo_bf16_to_f32(sh);
        if (!finite || !isfinite(shf)) {
            status |= HQO_ST_NONFINITE;
            sh = 0;
            shf = 0.0f;
        } else if (shf < 1.2621774483536189e-29f /* 2^-96 */) {
            sh = 0;
            shf = 0.0f;
        }
        scale_out[r] = sh;
        if (shf == 0.0f) {
            for (int j = 0; j < n; ++j) u_out[r * n + j] = 0.0f;
            continue;
        }
        float g = 1.0f / (shf * beta);
        for (int j = 0; j < n; ++j) {
            float acc = 0.0f;
            for (int i = 0; i < n; ++i) acc = fmaf(Q[j * n + i], xt[i], acc);
            u_out[r * n + j] = acc * g;
        }
    }
    return status;
}

/*
 * Dense-rotation KV encode: x [rows, n] (rows = B*H*S head vectors of a [B, H, S, n] tensor,
 * row0 = global row of x's first row, tokens starting at kv_s0), codes with the KV dither of
 * row (b H + h, kv_s0 + s).  Outputs as hqo_encode with one tile column.
 */
uint32_t hqo_encode_dense(const void* x, int dtype, int64_t rows, int n, const float* Q, int lattice, float beta,
                          uint64_t seed, int64_t kv_S, int64_t row0, int64_t kv_s0, uint16_t* scale, uint16_t* meta,
                          uint32_t* chunk_word, uint32_t* bits, int64_t cap_words, int32_t* v_out, float* u_out)
{
    if (!valid_common(n, lattice) || n > 128 || rows <= 0 || kv_S <= 0 || kv_s0 < 0) return 1u << 1;
    float* u = (float*)malloc(sizeof(float) * (size_t)(rows * n));
    if (!u) return 1u << 1;
    uint32_t status = hqo_rotate_normalize(x, dtype, rows, n, Q, beta, u, scale);
    status |= quantize_rows(u, rows, n, lattice, 1, kv_S, row0, kv_s0, seed, v_out, meta, chunk_word, bits, cap_words);
    if (u_out) memcpy(u_out, u, sizeof(float) * (size_t)(rows * n));
    free(u);
    return status;
}

/* The lattice points of a code of rows x n normalised coefficients (one tile column) in u units,
 * minus the KV dither of row (b H + h, kv_s0 + s): E8 v/2, A2 (P/2, Q sqrt3/2), Z and D4 v, the
 * dither taken off in the quantizer's coordinates.  Binary64. */
uint32_t hqo_decode_coeffs(const uint16_t* meta, const uint32_t* chunk_word, const uint32_t* bits, int64_t rows, int n,
                           int lattice, uint64_t seed, int64_t kv_S, int64_t row0, int64_t kv_s0, double* p_out)
{
    if (!valid_common(n, lattice) || rows <= 0 || kv_S <= 0) return 1u << 1;
    int32_t* v = (int32_t*)malloc(sizeof(int32_t) * (size_t)(rows * n));
    if (!v) return 1u << 1;
    uint32_t status = hqo_parse(meta, chunk_word, bits, rows, n, n, lattice, v);
    for (int64_t r = 0; r < rows; ++r) {
        int64_t c1 = 0, cw = 0;
        dither_words(1, row0 + r, kv_S, kv_s0, 0, &c1, &cw);
        float U[HQO_MAXN];
        hqo_dither(lattice, seed, c1, cw, n, U);
        for (int i = 0; i < n; ++i) {
            const double vi = (double)v[r * n + i], Ui = (double)U[i];
            double p;
            if (lattice == HQO_E8) p = 0.5 * vi - Ui;
            else if (lattice == HQO_A2) p = (i & 1) ? (vi - Ui) * (sqrt(3.0) / 2.0) : 0.5 * (vi - Ui);
            else p = vi - Ui;
            p_out[r * n + i] = p;
        }
    }
    free(v);
    return status;
}

/* Inverse rotation: x_hat_i = (sum_j Q[j][i] p_j) (s_hat beta), i.e. Q^T p rescaled.  Binary64. */
void hqo_unrotate(const double* p, const uint16_t* scale, int64_t rows, int n, const float* Q, float beta, double* out)
{
    for (int64_t r = 0; r < rows; ++r) {
        const double h = (double)hqo_bf16_to_f32(scale[r]) * (double)beta;
        for (int i = 0; i < n; ++i) {
            double acc = 0.0;
            for (int j = 0; j < n; ++j) acc += (double)Q[j * n + i] * p[r * n + j];
            out[r * n + i] = acc * h;
        }
    }
}

/* Dense-rotation KV decode to binary64 out[rows, n]. */
uint32_t hqo_decode_dense(const uint16_t* scale, const uint16_t* meta, const uint32_t* chunk_word, const uint32_t* bits,
                          int64_t rows, int n, const float* Q, int lattice, float beta, uint64_t seed, int64_t kv_S,
                          int64_t row0, int64_t kv_s0, double* out)
{
    double* p = (double*)malloc(sizeof(double) * (size_t)(rows > 0 ? rows * n : 1));
    if (!p) return 1u << 1;
    uint32_t status = hqo_decode_coeffs(meta, chunk_word, bits, rows, n, lattice, seed, kv_S, row0, kv_s0, p);
    if (!(status & 2u)) hqo_unrotate(p, scale, rows, n, Q, beta, out);
    free(p);
    return status;
}
