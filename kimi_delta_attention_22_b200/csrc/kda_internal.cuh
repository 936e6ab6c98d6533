// kda_internal.cuh -- launch interfaces shared by the host API and the kernels
// of libkda.  Not part of the public ABI (that is include/kda.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kda.h"
#include "kda_chunk_record.cuh"

namespace kda {

// Everything a chunked-prefill launch needs, already validated on the host.
struct ChunkArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    const float* S0;
    const int32_t* cu_seqlens;  // nullptr: dense batch, sequence n = rows [n*T, (n+1)*T)
    void* out;
    float* S_T;
    int32_t* dev_status;
    int B, T, H, d_k, d_v, num_seqs, gate, chunk;
    int Hk;       // query/key heads: value head h reads q/k head h / (H / Hk)
    float scale;  // d_k^{-1/2}
};

struct DecodeArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    float* S;
    void* out;
    int N, H, d_k, d_v, gate;
    int Hk;       // query/key heads: value head h reads q/k head h / (H / Hk)
    float scale;
};

// Multi-token recurrent pass (dense batch: N sequences of T tokens each).
struct RecurrentArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    float* S;
    void* out;
    int N, T, H, d_k, d_v, gate;
    int Hk;       // query/key heads: value head h reads q/k head h / (H / Hk)
    float scale;
};

// Gradients of the token loop (dense batch, as RecurrentArgs); dq, dk, dg, dbeta are
// accumulated with atomics into zeroed buffers, dv and dS0 written.
struct RecurrentBwdArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    const float* S0;      // may be null (zero state)
    const void* d_out;
    const float* d_ST;    // may be null (zero)
    float* dq;
    float* dk;
    float* dv;
    float* dg;            // null without a gate
    float* dbeta;
    float* dS0;           // may be null
    float* ws;            // recurrent_bwd_workspace_bytes()
    int N, T, H, Hk, d_k, d_v, gate;
    float scale;
};

cudaError_t launch_recurrent(const RecurrentArgs& a, bool bf16, cudaStream_t s);
cudaError_t launch_recurrent_bwd(const RecurrentBwdArgs& a, bool bf16, cudaStream_t s);
size_t recurrent_bwd_workspace_bytes(int N, int T, int H, int d_v);
cudaError_t launch_chunk_f32path(const ChunkArgs& a, bool bf16, cudaStream_t s);
// Two-kernel tensor-core prefill over a caller workspace laid out by rec::layout().
cudaError_t launch_chunk_wy(const ChunkArgs& a, uint8_t* ws, const rec::Layout& lay, cudaStream_t s);
// S_chk: null, or [slot][H][d_v][d_k] fp32 to receive the incoming state of every chunk
// (the backward's checkpoints); a.out may then be null (no outputs written).
cudaError_t launch_chunk_scan(const ChunkArgs& a, const uint8_t* ws, const rec::Layout& lay,
                              cudaStream_t s, float* S_chk = nullptr);
cudaError_t launch_decode(const DecodeArgs& a, bool bf16, cudaStream_t s);
// One CTA taking the kernels' bounded mbarrier wait (budget_ns) on a barrier that
// completes (complete) or never does; on expiry it ORs KDA_DEV_TIMEOUT into *dev_status.
cudaError_t launch_selftest_wait(int32_t* dev_status, uint64_t budget_ns, bool complete, cudaStream_t s);

// Rows [bos, eos) of the packed token axis that sequence n covers.  Returns
// false (and flags dev_status) when cu_seqlens is inconsistent.
__device__ __forceinline__ bool seq_bounds(const int32_t* cu, int n, int T, int num_seqs,
                                           int32_t* dev_status, long long& bos,
                                           long long& eos) {
    if (cu == nullptr) {
        bos = (long long)n * T;
        eos = bos + T;
        return true;
    }
    const int a = cu[n], b = cu[n + 1];
    if (a < 0 || b < a || b > T || (n == 0 && a != 0)) {
        if (dev_status && threadIdx.x == 0) atomicOr(dev_status, KDA_DEV_BAD_SEQLENS);
        return false;
    }
    bos = a;
    eos = b;
    return true;
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

}  // namespace kda
