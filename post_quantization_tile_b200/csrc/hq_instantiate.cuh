// hq_instantiate.cuh -- grid sizing and template dispatch for one lattice, included by the
// per-lattice translation units hq_inst_<lattice>.cu (which define HQ_LAT, HQ_ENC, HQ_DEC).
#pragma once
#include "hq_decode.cuh"
#include "hq_encode.cuh"
#include "hq_launch.h"

namespace hq {

// persistent grid: the blocks that fit on the GPU at once (a multiple of the SM count), never
// more than the number of items
template <typename Args>
static cudaError_t launch_persistent(void (*kernel)(Args, CUtensorMap), size_t smem, int64_t items,
                                     const Args& a, const CUtensorMap& m, cudaStream_t st)
{
    cudaError_t e = cudaFuncSetAttribute((const void*)kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, (const void*)kernel, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    int64_t grid = (int64_t)per_sm * num_sms();
    if (grid > items) grid = items;
    if (grid < 1) grid = 1;
    kernel<<<(unsigned)grid, kThreads, smem, st>>>(a, m);
    return cudaGetLastError();
}

template <int N, int LAT, bool KV, int SRC, bool COUNT>
static cudaError_t enc_one(const EncodeArgs& a, const CUtensorMap& m, cudaStream_t st)
{
    return launch_persistent<EncodeArgs>(encode_kernel<N, LAT, KV, SRC, COUNT>, sizeof(EncSmem<N, SRC>) + 1024, a.items, a, m, st);
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

template <int N, int LAT, bool KV, int DST>
static cudaError_t dec_one(const DecodeArgs& a, const CUtensorMap& m, cudaStream_t st)
{
    return launch_persistent<DecodeArgs>(decode_kernel<N, LAT, KV, DST>, sizeof(DecSmem<N, DST>) + 1024, a.items, a, m, st);
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
    cudaError_t launch_decode_##SUFFIX(int n, bool kv, int dst, const DecodeArgs& a, const CUtensorMap& m,  \
                                       cudaStream_t st)                                                     \
    {                                                                                                       \
        return dec_dispatch<LAT>(n, kv, dst, a, m, st);                                                     \
    }                                                                                                       \
    }
