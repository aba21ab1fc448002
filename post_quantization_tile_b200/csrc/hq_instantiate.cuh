// hq_instantiate.cuh -- grid sizing and template dispatch for one lattice, included by the
// per-lattice translation units hq_inst_<lattice>.cu (which define HQ_LAT, HQ_ENC, HQ_DEC).
#pragma once
#include "hq_decode.cuh"
#include "hq_encode.cuh"
#include "hq_launch.h"

namespace hq {

static_assert(kEncodeBatchMax == kEncodeBatchMaxL, "batch size of the launch declarations");

// persistent grid: the blocks that fit on the GPU at once (a multiple of the SM count), never
// more than the number of items
static cudaError_t persistent_grid(const void* kernel, size_t smem, int64_t items, int64_t& grid)
{
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    grid = (int64_t)per_sm * num_sms();
    if (grid > items) grid = items;
    if (grid < 1) grid = 1;
    return cudaSuccess;
}

template <typename Args>
static cudaError_t launch_persistent(void (*kernel)(Args, CUtensorMap), size_t smem, int64_t items,
                                     const Args& a, const CUtensorMap& m, cudaStream_t st)
{
    int64_t grid = 0;
    const cudaError_t e = persistent_grid((const void*)kernel, smem, items, grid);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)grid, kThreads, smem, st>>>(a, m);
    return cudaGetLastError();
}

template <int N, int LAT, bool KV, int SRC, bool COUNT, int MAXB>
static cudaError_t enc_batch(const EncodeBatch<MAXB>& b, cudaStream_t st)
{
    const void* k = (const void*)encode_kernel<N, LAT, KV, SRC, COUNT, MAXB>;
    int64_t grid = 0;
    const cudaError_t e = persistent_grid(k, sizeof(EncSmem<N, SRC>) + 1024, b.item0[b.count], grid);
    if (e != cudaSuccess) return e;
    encode_kernel<N, LAT, KV, SRC, COUNT, MAXB><<<(unsigned)grid, kThreads, sizeof(EncSmem<N, SRC>) + 1024, st>>>(b);
    return cudaGetLastError();
}

template <int N, int LAT, bool KV, int SRC, bool COUNT>
static cudaError_t enc_one(const EncodeArgs& a, const CUtensorMap& m, cudaStream_t st)
{
    EncodeBatch<1> b;
    b.map[0] = m;
    b.arg[0] = a;
    b.item0[0] = 0;
    b.item0[1] = a.items;
    b.count = 1;
    return enc_batch<N, LAT, KV, SRC, COUNT, 1>(b, st);
}

// several weight tensors (no dither, bf16 or fp32) in one launch; KV tensors (with the dither) of
// head dimension 128
template <int LAT>
static cudaError_t enc_batch_dispatch(int n, bool kv, int src, const EncodeBatch<kEncodeBatchMax>& b, cudaStream_t st)
{
    if (kv) {
        if (n != 128) return cudaErrorInvalidValue;
        return src == 0 ? enc_batch<128, LAT, true, 0, false, kEncodeBatchMax>(b, st)
                        : enc_batch<128, LAT, true, 1, false, kEncodeBatchMax>(b, st);
    }
    if (src == 0) {
        if (n == 64) return enc_batch<64, LAT, false, 0, false, kEncodeBatchMax>(b, st);
        if (n == 128) return enc_batch<128, LAT, false, 0, false, kEncodeBatchMax>(b, st);
        return enc_batch<256, LAT, false, 0, false, kEncodeBatchMax>(b, st);
    }
    if (src == 1) {
        if (n == 64) return enc_batch<64, LAT, false, 1, false, kEncodeBatchMax>(b, st);
        if (n == 128) return enc_batch<128, LAT, false, 1, false, kEncodeBatchMax>(b, st);
    }
    return cudaErrorInvalidValue;
}

template <int N, int LAT, bool KV, int SRC>
static cudaError_t enc_count(bool count, const EncodeArgs& a, const CUtensorMap& m, cudaStream_t st)
{
    if constexpr (SRC == 2) {
        return count ? cudaErrorInvalidValue : enc_one<N, LAT, KV, SRC, false>(a, m, st);
    } else {
        return count ? enc_one<N, LAT, KV, SRC, true>(a, m, st) : enc_one<N, LAT, KV, SRC, false>(a, m, st);
    }
}

template <int N, int LAT, bool KV>
static cudaError_t enc_src(int src, bool count, const EncodeArgs& a, const CUtensorMap& m, cudaStream_t st)
{
    if (src == 0) return enc_count<N, LAT, KV, 0>(count, a, m, st);
    if (src == 2) return enc_count<N, LAT, KV, 2>(count, a, m, st);
    if constexpr (N == 256) {
        return cudaErrorInvalidValue;  // fp32 weights use tiles of at most 128
    } else {
        return enc_count<N, LAT, KV, 1>(count, a, m, st);
    }
}

template <int LAT>
static cudaError_t enc_dispatch(int n, bool kv, int src, bool count, const EncodeArgs& a, const CUtensorMap& m,
                                cudaStream_t st)
{
    if (kv) {  // with the subtractive dither
        if (n == 64) return enc_src<64, LAT, true>(src, count, a, m, st);
        if (n == 128) return enc_src<128, LAT, true>(src, count, a, m, st);
        return enc_src<256, LAT, true>(src, count, a, m, st);
    }
    if (n == 64) return enc_src<64, LAT, false>(src, count, a, m, st);
    if (n == 128) return enc_src<128, LAT, false>(src, count, a, m, st);
    return enc_src<256, LAT, false>(src, count, a, m, st);
}

template <int N, int LAT, bool KV, int DST, int MAXB>
static cudaError_t dec_batch(const DecodeBatch<MAXB>& b, cudaStream_t st)
{
    const void* k = (const void*)decode_kernel<N, LAT, KV, DST, MAXB>;
    int64_t grid = 0;
    const cudaError_t e = persistent_grid(k, sizeof(DecSmem<N, DST>) + 1024, b.item0[b.count], grid);
    if (e != cudaSuccess) return e;
    decode_kernel<N, LAT, KV, DST, MAXB><<<(unsigned)grid, kThreads, sizeof(DecSmem<N, DST>) + 1024, st>>>(b);
    return cudaGetLastError();
}

template <int N, int LAT, bool KV, int DST>
static cudaError_t dec_one(const DecodeArgs& a, const CUtensorMap& m, cudaStream_t st)
{
    DecodeBatch<1> b;
    b.map[0] = m;
    b.arg[0] = a;
    b.item0[0] = 0;
    b.item0[1] = a.items;
    b.count = 1;
    return dec_batch<N, LAT, KV, DST, 1>(b, st);
}

// several weight codes (no dither) to bf16 or fp32 in one launch
template <int LAT>
static cudaError_t dec_batch_dispatch(int n, int dst, const DecodeBatch<kEncodeBatchMax>& b, cudaStream_t st)
{
    if (dst == 0) {
        if (n == 64) return dec_batch<64, LAT, false, 0, kEncodeBatchMax>(b, st);
        if (n == 128) return dec_batch<128, LAT, false, 0, kEncodeBatchMax>(b, st);
        return dec_batch<256, LAT, false, 0, kEncodeBatchMax>(b, st);
    }
    if (dst == 1) {
        if (n == 64) return dec_batch<64, LAT, false, 1, kEncodeBatchMax>(b, st);
        if (n == 128) return dec_batch<128, LAT, false, 1, kEncodeBatchMax>(b, st);
        return dec_batch<256, LAT, false, 1, kEncodeBatchMax>(b, st);
    }
    return cudaErrorInvalidValue;
}

template <int N, int LAT, bool KV>
static cudaError_t dec_dst(int dst, const DecodeArgs& a, const CUtensorMap& m, cudaStream_t st)
{
    if (dst == 2) {  // int8 lattice codes: integer-valued lattices without dither, 128-byte tile rows
        if constexpr (!KV && LAT != HQ_A2 && N != 64) return dec_one<N, LAT, KV, 2>(a, m, st);
        return cudaErrorInvalidValue;
    }
    if (dst == 3) {  // dithered lattice points for the dense inverse rotation: KV tiles of 128
        if constexpr (KV && N == 128) return dec_one<N, LAT, KV, 3>(a, m, st);
        return cudaErrorInvalidValue;
    }
    return dst == 0 ? dec_one<N, LAT, KV, 0>(a, m, st) : dec_one<N, LAT, KV, 1>(a, m, st);
}

template <int LAT>
static cudaError_t dec_dispatch(int n, bool kv, int dst, const DecodeArgs& a, const CUtensorMap& m, cudaStream_t st)
{
    if (kv) {  // with the subtractive dither
        if (n == 64) return dec_dst<64, LAT, true>(dst, a, m, st);
        if (n == 128) return dec_dst<128, LAT, true>(dst, a, m, st);
        return dec_dst<256, LAT, true>(dst, a, m, st);
    }
    if (n == 64) return dec_dst<64, LAT, false>(dst, a, m, st);
    if (n == 128) return dec_dst<128, LAT, false>(dst, a, m, st);
    return dec_dst<256, LAT, false>(dst, a, m, st);
}

}  // namespace hq

#define HQ_DEFINE_LAUNCHERS(LAT, SUFFIX)                                                                    \
    namespace hq {                                                                                          \
    cudaError_t launch_encode_##SUFFIX(int n, bool kv, int src, bool count, const EncodeArgs& a,           \
                                       const CUtensorMap& m, cudaStream_t st)                               \
    {                                                                                                       \
        return enc_dispatch<LAT>(n, kv, src, count, a, m, st);                                              \
    }                                                                                                       \
    cudaError_t launch_encode_batch_##SUFFIX(int n, bool kv, int src, const EncodeBatch<kEncodeBatchMax>& b, \
                                             cudaStream_t st)                                               \
    {                                                                                                       \
        return enc_batch_dispatch<LAT>(n, kv, src, b, st);                                                  \
    }                                                                                                       \
    cudaError_t launch_decode_##SUFFIX(int n, bool kv, int dst, const DecodeArgs& a, const CUtensorMap& m,  \
                                       cudaStream_t st)                                                     \
    {                                                                                                       \
        return dec_dispatch<LAT>(n, kv, dst, a, m, st);                                                     \
    }                                                                                                       \
    cudaError_t launch_decode_batch_##SUFFIX(int n, int dst, const DecodeBatch<kEncodeBatchMax>& b,          \
                                             cudaStream_t st)                                               \
    {                                                                                                       \
        return dec_batch_dispatch<LAT>(n, dst, b, st);                                                      \
    }                                                                                                       \
    }
