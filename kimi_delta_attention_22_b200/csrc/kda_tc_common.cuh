// kda_tc_common.cuh -- element packing, fast exponentials, warp-level tf32
// 16x16 block products and TMA tensor-map construction shared by the
// tensor-core chunk kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "sm100.cuh"

namespace kda {
namespace tc {

using namespace sm100;

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&t);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    __nv_bfloat162 t = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(t);
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    __half2 t = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&t);
}
__device__ __forceinline__ float2 unpack_f16(uint32_t u) {
    __half2 t = *reinterpret_cast<__half2*>(&u);
    return __half22float2(t);
}
__device__ __forceinline__ void st_shared_v4(uint8_t* base, uint32_t off, uint4 v) {
    *reinterpret_cast<uint4*>(base + off) = v;
}

constexpr float kLog2e = 1.4426950408889634f;

// 2^x on the special-function unit (inputs here are differences of
// cumulative log2 decays, so |x| stays far below the exponent range).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// acc (16x16, two m16n8 C fragments) += A (16x16) * B (16x16), both fp32 in
// shared memory (row-major, strides lda / ldb), on the warp-level tf32 MMA.
__device__ __forceinline__ void blk_mma(float (&acc)[2][4], const float* A, int lda, const float* B,
                                        int ldb, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const uint32_t a0 = to_tf32(A[g * lda + 8 * ks + t]);
        const uint32_t a1 = to_tf32(A[(g + 8) * lda + 8 * ks + t]);
        const uint32_t a2 = to_tf32(A[g * lda + 8 * ks + t + 4]);
        const uint32_t a3 = to_tf32(A[(g + 8) * lda + 8 * ks + t + 4]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const uint32_t b0 = to_tf32(B[(8 * ks + t) * ldb + 8 * nt + g]);
            const uint32_t b1 = to_tf32(B[(8 * ks + t + 4) * ldb + 8 * nt + g]);
            asm volatile(
                "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, "
                "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
                : "+f"(acc[nt][0]), "+f"(acc[nt][1]), "+f"(acc[nt][2]), "+f"(acc[nt][3])
                : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
        }
    }
}

// K-major view (K = channel) of rows laid out by mnmaj_off(c, row, 128): k-step s.
__device__ __forceinline__ uint64_t rowview_desc(uint32_t base, int s) {
    return desc_sw128(base + (uint32_t)((s >> 2) * 1024 + (s & 3) * 32), 16, 2048);
}

// As blk_mma with A = s0 A0 + s1 A1 (+ s2 A2 when A2 is not null), all stride lda.
__device__ __forceinline__ void blk_mma2(float (&acc)[2][4], const float* A0, float s0,
                                         const float* A1, float s1, const float* A2, float s2,
                                         int lda, const float* B, int ldb, int lane) {
    const int g = lane >> 2, t = lane & 3;
    auto av = [&](int off) {
        float x = s0 * A0[off] + s1 * A1[off];
        if (A2) x += s2 * A2[off];
        return to_tf32(x);
    };
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const uint32_t a0 = av(g * lda + 8 * ks + t);
        const uint32_t a1 = av((g + 8) * lda + 8 * ks + t);
        const uint32_t a2 = av(g * lda + 8 * ks + t + 4);
        const uint32_t a3 = av((g + 8) * lda + 8 * ks + t + 4);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const uint32_t b0 = to_tf32(B[(8 * ks + t) * ldb + 8 * nt + g]);
            const uint32_t b1 = to_tf32(B[(8 * ks + t + 4) * ldb + 8 * nt + g]);
            asm volatile(
                "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, "
                "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
                : "+f"(acc[nt][0]), "+f"(acc[nt][1]), "+f"(acc[nt][2]), "+f"(acc[nt][3])
                : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
        }
    }
}

// Store a 16x16 C-fragment pair, scaled by s, to shared memory (row stride ld).
__device__ __forceinline__ void blk_store(float* Cm, int ld, const float (&acc)[2][4], int lane,
                                          float s) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        Cm[g * ld + 8 * nt + 2 * t] = s * acc[nt][0];
        Cm[g * ld + 8 * nt + 2 * t + 1] = s * acc[nt][1];
        Cm[(g + 8) * ld + 8 * nt + 2 * t] = s * acc[nt][2];
        Cm[(g + 8) * ld + 8 * nt + 2 * t + 1] = s * acc[nt][3];
    }
}

__device__ __forceinline__ void unpack8(uint4 u, float* f) {
    const float2 a = unpack_bf16(u.x), b = unpack_bf16(u.y), c = unpack_bf16(u.z), d = unpack_bf16(u.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y; f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

// Store 8 consecutive fp32 values as one 16-byte bf16 chunk.
__device__ __forceinline__ uint4 pack8(const float* v) {
    return make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                      pack_bf16(v[6], v[7]));
}

// 8 consecutive fp32 values as one 16-byte fp16 chunk, and back.
__device__ __forceinline__ uint4 pack8_f16(const float* v) {
    return make_uint4(pack_f16(v[0], v[1]), pack_f16(v[2], v[3]), pack_f16(v[4], v[5]),
                      pack_f16(v[6], v[7]));
}
__device__ __forceinline__ void unpack8_f16(uint4 u, float* f) {
    const float2 a = unpack_f16(u.x), b = unpack_f16(u.y), c = unpack_f16(u.z), d = unpack_f16(u.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y; f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}
// Two-term bf16 expansion of 8 fp32 values: hi = bf16(v), lo = bf16(v - hi), so that
// hi + lo carries about 16 significant bits (products of expansions summed in fp32
// keep the operand rounding near 2^-17 relative instead of bf16's 2^-9).
__device__ __forceinline__ void pack8_split(const float* v, uint4& hi, uint4& lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        h[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
        const float2 r = unpack_bf16(h[e]);   // exact: the rounded pair back in fp32
        l[e] = pack_bf16(v[2 * e] - r.x, v[2 * e + 1] - r.y);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Two-term fp16 expansion of 8 fp32 values: hi = fp16(v), lo = fp16(v - hi); hi + lo
// carries about 22 significant bits (lo's own rounding, or its underflow below fp16's
// normal range, bounds the rest).
__device__ __forceinline__ void pack8_split16(const float* v, uint4& hi, uint4& lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        h[e] = pack_f16(v[2 * e], v[2 * e + 1]);
        const float2 r = unpack_f16(h[e]);   // exact: the rounded pair back in fp32
        l[e] = pack_f16(v[2 * e] - r.x, v[2 * e + 1] - r.y);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// ------------------------------------------------------------------ host side

// Launch `kern` after the previous work of `st` with programmatic serialization:
// it may start (prologue) while that work drains and must call pdl_wait() before
// reading anything the previous kernel writes.
template <typename Params>
inline cudaError_t launch_after(void (*kern)(Params), dim3 grid, int block, int smem, cudaStream_t st,
                                const Params& prm) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, prm);
}

inline PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 3-D map over [tokens][H][width] (innermost first: width, H, tokens).
inline bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int width,
              int H, long long tokens, int box_w, int box_t, CUtensorMapSwizzle sw) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)width, (cuuint64_t)H, (cuuint64_t)tokens};
    cuuint64_t strides[2] = {(cuuint64_t)width * esize, (cuuint64_t)width * esize * H};
    cuuint32_t box[3] = {(cuuint32_t)box_w, 1u, (cuuint32_t)box_t};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace kda
