// hq_launch.h -- launchers of the encode / decode kernels, one translation unit per lattice.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/hq.h"

namespace hq {

struct EncodeArgs;
struct DecodeArgs;
template <int MAXB>
struct EncodeBatch;
template <int MAXB>
struct DecodeBatch;
constexpr int kEncodeBatchMaxL = 16;  // = kEncodeBatchMax (hq_encode.cuh)

// src: 0 bf16 weight, 1 fp32 weight, 2 fp32 normalised coefficients; count: count-only pass
cudaError_t launch_encode_z(int n, bool kv, int src, bool count, const EncodeArgs& a, const CUtensorMap& m, cudaStream_t st);
cudaError_t launch_encode_a2(int n, bool kv, int src, bool count, const EncodeArgs& a, const CUtensorMap& m, cudaStream_t st);
cudaError_t launch_encode_d4(int n, bool kv, int src, bool count, const EncodeArgs& a, const CUtensorMap& m, cudaStream_t st);
cudaError_t launch_encode_e8(int n, bool kv, int src, bool count, const EncodeArgs& a, const CUtensorMap& m, cudaStream_t st);
// several weight tensors (kv false), or KV tensors of head dimension 128 with the dither (kv true),
// of one tile size, lattice and source type in one launch
cudaError_t launch_encode_batch_z(int n, bool kv, int src, const EncodeBatch<kEncodeBatchMaxL>& b, cudaStream_t st);
cudaError_t launch_encode_batch_a2(int n, bool kv, int src, const EncodeBatch<kEncodeBatchMaxL>& b, cudaStream_t st);
cudaError_t launch_encode_batch_d4(int n, bool kv, int src, const EncodeBatch<kEncodeBatchMaxL>& b, cudaStream_t st);
cudaError_t launch_encode_batch_e8(int n, bool kv, int src, const EncodeBatch<kEncodeBatchMaxL>& b, cudaStream_t st);
// several weight codes of one tile size and lattice to bf16 (dst 0) or fp32 (dst 1) in one launch
cudaError_t launch_decode_batch_z(int n, int dst, const DecodeBatch<kEncodeBatchMaxL>& b, cudaStream_t st);
cudaError_t launch_decode_batch_a2(int n, int dst, const DecodeBatch<kEncodeBatchMaxL>& b, cudaStream_t st);
cudaError_t launch_decode_batch_d4(int n, int dst, const DecodeBatch<kEncodeBatchMaxL>& b, cudaStream_t st);
cudaError_t launch_decode_batch_e8(int n, int dst, const DecodeBatch<kEncodeBatchMaxL>& b, cudaStream_t st);
// dst: 0 bf16, 1 fp32, 2 int8 codes, 3 fp32 lattice points minus the dither (u units)
cudaError_t launch_decode_z(int n, bool kv, int dst, const DecodeArgs& a, const CUtensorMap& m, cudaStream_t st);
cudaError_t launch_decode_a2(int n, bool kv, int dst, const DecodeArgs& a, const CUtensorMap& m, cudaStream_t st);
cudaError_t launch_decode_d4(int n, bool kv, int dst, const DecodeArgs& a, const CUtensorMap& m, cudaStream_t st);
cudaError_t launch_decode_e8(int n, bool kv, int dst, const DecodeArgs& a, const CUtensorMap& m, cudaStream_t st);

int num_sms();

// dense-rotation KV variant (hq_dense.cu): forward rotation to normalised coefficients, inverse
// rotation of decoded lattice points, and the forward pass's non-finite count into the status word
cudaError_t launch_rotate(const void* x, bool bf16, const float* Q, float beta, int64_t rows, float* u,
                          uint16_t* scale, uint32_t* nonfinite, cudaStream_t st);
cudaError_t launch_unrotate(const float* p, const float* Q, const uint16_t* scale, float beta, int64_t rows, void* y,
                            bool bf16, void* ws, cudaStream_t st);
cudaError_t launch_merge_nonfinite(void* ws, const uint32_t* nonfinite, cudaStream_t st);

// 2-D tensor map of a row-major [rows, cols] tensor of es-byte elements: box [box_rows][128 bytes],
// 128-byte swizzle (hq_api.cu)
bool tensor_map_2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int es, int box_rows);
// make the device that owns p current (hq_api.cu)
bool device_of(const void* p);
// workspace bytes of the encoder for one source (0 bf16, 1 fp32 weights, 2 coefficients); 0 if
// the shape is invalid (hq_api.cu)
size_t encode_workspace_bytes(int64_t rows, int64_t cols, int32_t n, int src);

}  // namespace hq
