// common.cuh -- helpers shared by the library's CUDA translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "iqq.h"

namespace iqq {

// The cudaError_t of the last failed launch on this host thread.
void set_last_cuda_error(cudaError_t e);

// Maps the launch result to a status, remembering a failure.
inline iqq_status launch_status()
{
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_last_cuda_error(e);
        return IQQ_ERR_CUDA;
    }
    return IQQ_OK;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// nrows * n_per_row * bytes_per_value fits in int64.
inline bool size_ok(int64_t nrows, int64_t n_per_row, int64_t bytes_per_value)
{
    if (nrows < 0 || n_per_row < 0) return false;
    if (nrows == 0 || n_per_row == 0) return true;
    return nrows <= INT64_MAX / n_per_row / bytes_per_value;
}

// Streaming 16-byte load that bypasses L1 allocation (data read once).
__device__ __forceinline__ float4 ld_stream_f4(const float4* p)
{
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

// Four bf16 values (little endian in two words) widened to binary32: a bf16 is the high
// half of the binary32 with the same value, so the widening is exact.
__device__ __forceinline__ float4 widen_bf16x4(uint2 v)
{
    return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                       __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
}

// Values p[0..3] as binary32, from binary32 storage (p 16-byte aligned) or bf16 storage
// (p 8-byte aligned); read-only path.
__device__ __forceinline__ float4 ld4(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16* p)
{
    return widen_bf16x4(__ldg(reinterpret_cast<const uint2*>(p)));
}

// The same, streaming (no L1 allocation: data read once).
__device__ __forceinline__ float4 ld4_stream(const float* p) { return ld_stream_f4(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ float4 ld4_stream(const __nv_bfloat16* p)
{
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return widen_bf16x4(v);
}

// Flags word update: only lanes with a nonzero bit set touch memory.
__device__ __forceinline__ void raise_flags(uint32_t* flags, uint32_t bits)
{
    if (flags != nullptr && bits != 0u) atomicOr(flags, bits);
}

// The Q4_0 weighted quantizer with the transition-based sweep (q4_0_w.cu): rows of fewer
// than 2^22 blocks; binary32 x may also take the epilogue outputs (y_out: the dequantized
// values; acc: the round-trip accumulator), each optional.
bool q4_0_w_fits(int64_t n_per_row);
iqq_status launch_q4_0_w(const float* x, const float* qw, void* out, int64_t nrows, int64_t n_per_row,
                         int64_t rows_per_qw, int weight_mode, float fudge, uint32_t* d_flags, void* stream,
                         float* y_out = nullptr, double* acc = nullptr);
iqq_status launch_q4_0_w(const __nv_bfloat16* x, const float* qw, void* out, int64_t nrows, int64_t n_per_row,
                         int64_t rows_per_qw, int weight_mode, float fudge, uint32_t* d_flags, void* stream);
// Several binary32 tensors, validated by the caller, in launches of up to 64 tensors.
iqq_status launch_q4_0_w_batch(const iqq_q4_0_problem* probs, int64_t count, int weight_mode, float fudge,
                               uint32_t* d_flags, void* stream);

}  // namespace iqq
