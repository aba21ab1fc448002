// hq_common.cuh -- device helpers shared by the encode and decode kernels of the HyperQuant
// tile codec: tile geometry, Philox4x32-10, TMA / mbarrier wrappers, bit writer and reader.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hq.h"

namespace hq {

// ------------------------------------------------------------------------------------------------
// Kernel configuration
// ------------------------------------------------------------------------------------------------
#ifndef HQ_QUANT_ROT
#define HQ_QUANT_ROT 4  // rounds of the quantizer body per tile (encode_kernel); 2 and 8 measured slower
#endif
#ifndef HQ_THREADS
#define HQ_THREADS 128
#endif
constexpr int kThreads = HQ_THREADS;   // threads per block (one tile row each, two for n = 256)
#ifndef HQ_MIN_BLOCKS
#define HQ_MIN_BLOCKS (384 / HQ_THREADS)
#endif
constexpr int kMinBlocks = HQ_MIN_BLOCKS;  // resident blocks per SM the register budget aims at
constexpr int kChunkTiles = 32;        // tiles per chunk (one warp scan)
constexpr int kStages = 2;             // input pipeline depth
constexpr uint32_t kSpinLimit = 1u << 22;  // bounded waits: polls before giving up

// status word bits (1 << hq_status_t)
constexpr uint32_t kStCapacity = 1u << HQ_ERR_CAPACITY;
constexpr uint32_t kStNonfinite = 1u << HQ_ERR_NONFINITE;
constexpr uint32_t kStCorrupt = 1u << HQ_ERR_CORRUPT;
constexpr uint32_t kStTimeout = 1u << HQ_ERR_TIMEOUT;
constexpr uint32_t kStRange = 1u << HQ_ERR_RANGE;

// Workspace layout (bytes): [0] status u32, [4] nonfinite tiles u32, [8] words needed u64,
// [16] work counter u32, [24] count-only total u64, [64 ..] look-back states u64 per item.
struct WsHeader {
    uint32_t status;
    uint32_t nonfinite;
    unsigned long long needed;
    uint32_t counter;
    uint32_t pad0;
    unsigned long long count_bits;
    uint32_t pad1[8];
};
static_assert(sizeof(WsHeader) == 64, "workspace header");

// Step search (exact-rate mode), kept in the workspace right after the header.  Count-only encodes
// read the probe step from here; a one-thread update kernel between them moves the bracket.
struct RateSearch {
    float probe;                   // step of the next count-only pass
    int32_t done;                  // 1: the search has ended, later passes return at once
    int32_t lo, hi;                // bracket as binary32 bit patterns (-1: side not seen yet)
    long long c_lo, c_hi;          // payload bits at lo (above target) and hi (at or below target)
    int32_t last_side;             // 0 none, 1 lo moved, 2 hi moved (last update)
    int32_t probes;                // count-only passes made
    int32_t best;                  // bits of the step with the smallest |bits - target| so far
    int32_t pad0;
    long long c_best;
    double target, tol;            // payload bits wanted, accepted distance
    double n;                      // scalars in the tensor
};
static_assert(sizeof(RateSearch) <= 192, "rate search state");

// threads per tile: one thread holds n/TPT coefficients in registers.  Two threads share a tile
// of 256 (256 registers of coefficients would not fit); for n = 128 the choice is a build option
// (the bit format does not depend on it).
#ifndef HQ_ENC_TPT128
#define HQ_ENC_TPT128 1
#endif
#ifndef HQ_DEC_TPT128
#define HQ_DEC_TPT128 1
#endif
#ifndef HQ_ENC_SEPARATE_ZZ
#define HQ_ENC_SEPARATE_ZZ 0
#endif
#ifndef HQ_DEC_STAGES
#define HQ_DEC_STAGES 1
#endif
// fp32 coefficients at n = 128: two threads per tile halve the TMA stage (64 rows of 512 bytes),
// so three blocks fit an SM instead of two
#ifndef HQ_ENC_TPT128_COEF
#define HQ_ENC_TPT128_COEF 2
#endif
// src: 0 bf16 weight, 1 fp32 weight, 2 fp32 coefficients (fp32 weights keep one thread per tile)
__host__ __device__ constexpr int enc_tpt(int n, int src)
{
    return (n == 256 || (n == 128 && ((src == 0 && HQ_ENC_TPT128 == 2) || (src == 2 && HQ_ENC_TPT128_COEF == 2))))
               ? 2
               : 1;
}
// the most threads per tile any encoder source uses (the workspace holds one look-back slot per item)
__host__ __device__ constexpr int enc_tpt_max(int n)
{
    return enc_tpt(n, 0) > enc_tpt(n, 2) ? enc_tpt(n, 0) : enc_tpt(n, 2);
}
__host__ __device__ constexpr int dec_tpt(int n) { return (n == 256 || (n == 128 && HQ_DEC_TPT128 == 2)) ? 2 : 1; }

// ------------------------------------------------------------------------------------------------
// Philox4x32-10 (Salmon et al., SC'11): published multipliers and Weyl key increments.
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1)
{
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint32_t lo0 = 0xD2511F53u * c.x;
        const uint32_t hi0 = __umulhi(0xD2511F53u, c.x);
        const uint32_t lo1 = 0xCD9E8D57u * c.z;
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z);
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    }
    return c;
}

// round keys of a 64-bit seed: rk[2 r], rk[2 r + 1] are the key words of round r
__host__ __device__ inline void philox_round_keys(uint64_t seed, uint32_t (&rk)[20])
{
    uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
    for (int r = 0; r < 10; ++r) {
        rk[2 * r] = k0;
        rk[2 * r + 1] = k1;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
}

// the same generator with precomputed round keys (kernel parameters: no registers held for them)
__device__ __forceinline__ uint4 philox4x32_10_rk(uint4 c, const uint32_t (&rk)[20])
{
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t lo0 = 0xD2511F53u * c.x;
        const uint32_t hi0 = __umulhi(0xD2511F53u, c.x);
        const uint32_t lo1 = 0xCD9E8D57u * c.z;
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z);
        c = make_uint4(hi1 ^ c.y ^ rk[2 * r], lo1, hi0 ^ c.w ^ rk[2 * r + 1], lo0);
    }
    return c;
}

// ------------------------------------------------------------------------------------------------
// bf16 / fp32 bit helpers
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// binary32 -> bfloat16 bits, round to nearest even (finite inputs)
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f)
{
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ float2 f2add(float2 a, float2 b) { return __fadd2_rn(a, b); }
// a - b as a fused multiply-add with an exact product: one rounding, like the subtraction
__device__ __forceinline__ float2 f2sub(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a); }
__device__ __forceinline__ float2 f2mul(float2 a, float2 b) { return __fmul2_rn(a, b); }

// ------------------------------------------------------------------------------------------------
// shared-memory, mbarrier and TMA wrappers
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// bounded wait on an mbarrier phase; returns false when the limit ran out
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity)
{
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if (i > 64) __nanosleep(64);
    }
    return false;
}

// 2-D tiled TMA load of one box into shared memory, completing on `bar`
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// 2-D tiled TMA store of one box from shared memory (bulk group)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int x, int y, const void* src)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(src))
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// wait until every committed bulk store has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// wait until every committed bulk store has completed
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// make generic-proxy shared-memory writes visible to the async (TMA) proxy
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 1-D bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16)
__device__ __forceinline__ void bulk_load_1d(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p)
{
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v)
{
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// address of byte `off` of row r inside a swizzled TMA box ([rows][128 B], 128-byte swizzle)
__device__ __forceinline__ uint32_t swz(int r, int chunk16) { return (uint32_t)(r * 128 + ((chunk16 ^ (r & 7)) << 4)); }

// ------------------------------------------------------------------------------------------------
// Bit writer.  Codes are appended in reading order into an MSB-first accumulator; full 32-bit
// reading-order words go to the shared-memory stream.  Forward segments read with increasing
// bit position (stored word = bit-reversed reading word), backward segments with decreasing
// position (stored word = reading word).  The accumulator starts with the phantom bits that
// precede the segment inside its first word, so every emitted word is one stored word.  The
// first and the last word of a segment may be shared with a neighbouring segment and are ORed
// atomically; the words in between belong to this segment alone.
// ------------------------------------------------------------------------------------------------
template <bool FWD>
struct BitWriter {
    unsigned long long acc;  // valid bits are the low `nb` bits, earliest read bit highest
    int nb;
    int wi;                  // stored word index of the next emitted word
    int wi0;                 // word index of the first (head) word
    uint32_t head;           // the head word, merged into the stream by finish()
    bool first;
    uint32_t* stg;

    __device__ __forceinline__ void begin(uint32_t* s, int start_or_end_bit)
    {
        stg = s;
        acc = 0ull;
        wi = start_or_end_bit >> 5;
        wi0 = wi;
        head = 0u;
        nb = FWD ? (start_or_end_bit & 31) : (31 - (start_or_end_bit & 31));
        first = true;
    }
    // The head word may share bits with a neighbouring tile (or the coset bits), so it is kept in
    // a register and OR-ed in by finish(); every later word belongs to this writer alone and is a
    // plain store.
    __device__ __forceinline__ void emit(uint32_t rw)
    {
        const uint32_t w = FWD ? __brev(rw) : rw;
        if (first) {
            head = w;
            first = false;
        } else {
            stg[wi] = w;
        }
        wi += FWD ? 1 : -1;
    }
    // append `len` (<= 32) bits: the low `len` bits of `code`, most significant first
    __device__ __forceinline__ void put(uint32_t code, int len)
    {
        acc = (acc << len) | code;
        nb += len;
        if (nb >= 32) {
            emit((uint32_t)(acc >> (nb - 32)));
            nb -= 32;
        }
    }
    // the partial last word and the head word meet other writers' bits: OR them in
    __device__ __forceinline__ void finish()
    {
        if (nb > 0) atomicOr(stg + wi, FWD ? __brev((uint32_t)(acc << (32 - nb))) : (uint32_t)(acc << (32 - nb)));
        if (!first) atomicOr(stg + wi0, head);
    }
};

// one Rice code of arbitrary length (long unary runs): the rare path, kept out of line
template <bool FWD>
__device__ __forceinline__ void put_long_code(BitWriter<FWD>& bw, uint32_t q, uint32_t code, int k)
{
    while (q > 31) {
        bw.put(0u, 31);
        q -= 31;
    }
    if (q) bw.put(0u, (int)q);
    bw.put(code, k + 1);
}

// Rice codes of four zig-zag values (reading order z0, z1, z2, z3): one append when their
// codes fit in 32 bits together, else one append per code
template <bool FWD>
__device__ __forceinline__ void put4(BitWriter<FWD>& bw, uint32_t z0, uint32_t z1, uint32_t z2, uint32_t z3, int k,
                                     uint32_t km, uint32_t one)
{
    const uint32_t q0 = z0 >> k, q1 = z1 >> k, q2 = z2 >> k, q3 = z3 >> k;
    const uint32_t c0 = (z0 & km) | one, c1 = (z1 & km) | one, c2 = (z2 & km) | one, c3 = (z3 & km) | one;
    const uint32_t k1 = (uint32_t)k + 1u;
    const uint32_t l0 = q0 + k1, l1 = q1 + k1, l2 = q2 + k1, l3 = q3 + k1;
    const uint32_t L = l0 + l1 + l2 + l3;
    if (L <= 32u) {
        // codes are (k+1)-bit values with the zero runs implied by the shifts; every partial
        // result has at most L <= 32 bits and every shift is at most 29, so 32 bits suffice
        uint32_t c = c0;
        c = (c << l1) | c1;
        c = (c << l2) | c2;
        c = (c << l3) | c3;
        bw.put(c, (int)L);
    } else {
        const uint32_t cs[4] = {c0, c1, c2, c3};
        const uint32_t qs[4] = {q0, q1, q2, q3};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (qs[j] + k1 <= 32u) bw.put(cs[j], (int)(qs[j] + k1));
            else put_long_code<FWD>(bw, qs[j], cs[j], k);
        }
    }
}

// ------------------------------------------------------------------------------------------------
// Bit reader over a shared-memory stream, mirror of BitWriter: MSB-aligned 64-bit window.
// ------------------------------------------------------------------------------------------------
template <bool FWD>
struct BitReader {
    unsigned long long W;  // top `avail` bits valid, next bit at bit 63
    int avail;
    int wi;
    int lim;  // last readable word index; reads are clamped to [0, lim]
    int c0;   // consumed() = 32 wi - avail - c0 (forward), c0 - 32 wi - avail (backward)
    const uint32_t* src;

    // bits taken from the stream since begin()
    __device__ __forceinline__ int consumed() const { return FWD ? 32 * wi - avail - c0 : c0 - 32 * wi - avail; }

    __device__ __forceinline__ uint32_t load()
    {
        const uint32_t w = src[min(max(wi, 0), lim)];
        wi += FWD ? 1 : -1;
        return FWD ? __brev(w) : w;
    }
    __device__ __forceinline__ void begin(const uint32_t* s, int start_or_end_bit, int last_word)
    {
        src = s;
        lim = last_word;
        wi = start_or_end_bit >> 5;
        const int skip = FWD ? (start_or_end_bit & 31) : (31 - (start_or_end_bit & 31));
        c0 = FWD ? 32 * wi + skip : 32 * wi - skip;
        const uint32_t w0 = load();
        const uint32_t w1 = load();
        W = (((unsigned long long)w0 << 32) | w1) << skip;
        avail = 64 - skip;
    }
    __device__ __forceinline__ void refill()
    {
        if (avail <= 32) {
            W |= (unsigned long long)load() << (32 - avail);
            avail += 32;
        }
    }
};

// unary runs of 32 or more zeros: the rare path, kept out of line.  Returns the run length
// beyond the first 32-bit head; clears ok past `limit`.
template <bool FWD>
__device__ __forceinline__ uint32_t long_run(BitReader<FWD>& br, uint32_t limit, bool& ok)
{
    uint32_t q = 0;
    uint32_t hi = (uint32_t)(br.W >> 32);
    while (hi == 0u) {
        q += 32;
        br.W <<= 32;
        br.avail -= 32;
        br.refill();
        hi = (uint32_t)(br.W >> 32);
        if (q > limit) {
            ok = false;
            return q;
        }
    }
    return q;
}

// the slow path of get_code (a code longer than the bits at hand, long unary runs), out of line:
// reader state in and out by value
struct RdOut {
    unsigned long long W;
    int avail, wi;
    uint32_t z;
    int ok;
};
template <bool FWD>
static __device__ __noinline__ RdOut get_code_slow(unsigned long long W, int avail, int wi, int lim, const uint32_t* src,
                                                   int k, uint32_t limit)
{
    BitReader<FWD> br;
    br.W = W;
    br.avail = avail;
    br.wi = wi;
    br.lim = lim;
    br.src = src;
    br.c0 = 0;
    bool ok = true;
    br.refill();
    uint32_t hi = (uint32_t)(br.W >> 32);
    uint32_t q = 0;
    RdOut o;
    if (hi == 0u) {
        q = long_run<FWD>(br, limit, ok);
        hi = (uint32_t)(br.W >> 32);
        if (!ok) {
            o.W = br.W; o.avail = br.avail; o.wi = br.wi; o.z = 0u; o.ok = 0;
            return o;
        }
    }
    const int z = __clz(hi);
    br.W <<= (z + 1);
    br.avail -= z + 1;
    if (br.avail < k) br.refill();
    const uint32_t r = k ? (uint32_t)(br.W >> (64 - k)) : 0u;
    br.W <<= k;
    br.avail -= k;
    q += (uint32_t)z;
    o.W = br.W; o.avail = br.avail; o.wi = br.wi; o.z = (q << k) | r; o.ok = 1;
    return o;
}

// one Rice code: q zeros, a one, r (k bits MSB-first); returns the zig-zag value q << k | r (the
// sum of q follows from the bits consumed: consumed() - codes (k + 1)).  The caller tops the window up to at least 33 bits every four codes;
// a code that is longer than the bits at hand takes the slow path (refill, long runs).
template <bool FWD>
__device__ __forceinline__ uint32_t get_code(BitReader<FWD>& br, int k, uint32_t pow2k, uint32_t limit, bool& ok)
{
    uint32_t hi = (uint32_t)(br.W >> 32);
    int z = __clz(hi);
    int lam = z + k + 1;
    if (hi == 0u || lam > br.avail) {
        const RdOut o = get_code_slow<FWD>(br.W, br.avail, br.wi, br.lim, br.src, k, limit);
        br.W = o.W;
        br.avail = o.avail;
        br.wi = o.wi;
        if (!o.ok) ok = false;
        return o.z;
    }
    // fast path: the whole code is in the top 32 bits: 0..0 1 r
    const uint32_t val = hi >> (32 - lam);      // (1 << k) | r
    br.W <<= lam;
    br.avail -= lam;
    return (uint32_t)z * pow2k + (val - pow2k);  // (z << k) | r
}

// ------------------------------------------------------------------------------------------------
// misc
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t zigzag(int32_t m) { return ((uint32_t)m << 1) ^ (uint32_t)(m >> 31); }
__device__ __forceinline__ int32_t unzigzag(uint32_t z) { return (int32_t)(z >> 1) ^ -(int32_t)(z & 1u); }

// Rice parameter: the smallest k >= 0 with sum zz < n 2^(k+1), capped at 15
__device__ __forceinline__ int rice_k(uint32_t A, int log2n)
{
    const uint32_t m = A >> (log2n + 1);
    const int k = 32 - __clz(m);
    return k > 15 ? 15 : k;
}

__device__ __forceinline__ void status_set(WsHeader* ws, uint32_t bits) { atomicOr(&ws->status, bits); }

}  // namespace hq
