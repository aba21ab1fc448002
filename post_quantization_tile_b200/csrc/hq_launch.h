// hq_launch.h -- launchers of the encode / decode kernels, one translation unit per lattice.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/hq.h"

namespace hq {

struct EncodeArgs;
struct DecodeArgs;

// src: 0 bf16 weight, 1 fp32 weight, 2 fp32 normalised coefficients; count: count-only pass
cudaError_t launch_encode_z(int n, bool kv, int src, bool count, const EncodeArgs& a, const CUtensorMap& m, cudaStream_t st);
cudaError_t launch_encode_a2(int n, bool kv, int src, bool count, const EncodeArgs& a, const CUtensorMap& m, cudaStream_t st);
cudaError_t launch_encode_d4(int n, bool kv, int src, bool count, const EncodeArgs& a, const CUtensorMap& m, cudaStream_t st);
cudaError_t launch_encode_e8(int n, bool kv, int src, bool count, const EncodeArgs& a, const CUtensorMap& m, cudaStream_t st);
// dst: 0 bf16, 1 fp32
cudaError_t launch_decode_z(int n, bool kv, int dst, const DecodeArgs& a, const CUtensorMap& m, cudaStream_t st);
cudaError_t launch_decode_a2(int n, bool kv, int dst, const DecodeArgs& a, const CUtensorMap& m, cudaStream_t st);
cudaError_t launch_decode_d4(int n, bool kv, int dst, const DecodeArgs& a, const CUtensorMap& m, cudaStream_t st);
cudaError_t launch_decode_e8(int n, bool kv, int dst, const DecodeArgs& a, const CUtensorMap& m, cudaStream_t st);

int num_sms();

// 2-D tensor map of a row-major [rows, cols] tensor of es-byte elements: box [box_rows][128 bytes],
// 128-byte swizzle (hq_api.cu)
bool tensor_map_2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int es, int box_rows);
// make the device that owns p current (hq_api.cu)
bool device_of(const void* p);

}  // namespace hq
