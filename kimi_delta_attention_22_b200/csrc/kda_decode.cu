// kda_decode.cu -- fused single-token KDA step (the recurrent schedule of the
// GeekNews summary of "You could have come up with Kimi Delta Attention",
// section "fused recurrent kernel for decode"; the five-step update at the
// top of the article).
//
// For one (sequence, head) with state S (d_v x d_k, row r = value index) and
// this token's q, k, v, alpha = exp(g), beta, every state row is independent:
//     sd_r  = S_r . Diag(alpha)                 (forget)
//     a_r   = sd_r . k,   b_r = sd_r . q~       (predict, and the pre-write read)
//     e_r   = beta (v_r - a_r)                  (correct)
//     S_r  <- sd_r + e_r k                      (write)
//     o_r   = b_r + e_r (k . q~)                (read of the post-write state)
// so the whole step is one pass over the state: each 512-byte row is read
// once and written once, and the two dot products are fused in registers.
//
// The step is HBM-bound (about 0.9 FLOP per byte of state traffic).  Layout
// of the work: a CTA owns 128 rows of one (n, h) state; each warp owns 16
// rows, four at a time, one row per 8-lane group; lane (l & 7) holds key
// columns 4(l & 7) + 32m, m = 0..3, so every 128-bit load instruction of a
// group covers one full 128-byte line of its row.  All 16 loads of a lane are
// issued before any arithmetic to keep 8 KB per warp in flight.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kDK = 128;           // key head size handled by this kernel
constexpr int kThreads = 256;      // 8 warps
constexpr int kRowsPerWarp = 16;
constexpr int kRowsPerCta = kRowsPerWarp * (kThreads / 32);

__device__ __forceinline__ void load4(const float* p, float* x) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(p));
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float* x) {
    const uint2 t = __ldg(reinterpret_cast<const uint2*>(p));
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&t.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&t.y);
    const float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}

template <typename TI, int GATE>
__global__ void __launch_bounds__(kThreads, 2) kda_decode_kernel(DecodeArgs a) {
    const int nh = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane & 7, rsel = lane >> 3;
    // query/key head of value head h = nh % H (grouped value heads share it)
    const size_t nhk = (size_t)(nh / a.H) * a.Hk + (nh % a.H) / (a.H / a.Hk);
    const TI* qp = static_cast<const TI*>(a.q) + nhk * kDK;
    const TI* kp = static_cast<const TI*>(a.k) + nhk * kDK;

    float kr[16], qr[16], al[16];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int c = 32 * m + 4 * sub;
        load4(kp + c, kr + 4 * m);
        load4(qp + c, qr + 4 * m);
        if (GATE == KDA_GATE_CHANNEL) {
            load4(a.g + (size_t)nh * kDK + c, al + 4 * m);
#pragma unroll
            for (int j = 0; j < 4; ++j) al[4 * m + j] = expf(al[4 * m + j]);
        }
    }
    if (GATE == KDA_GATE_SCALAR) {
        const float s = expf(__ldg(a.g + nh));
#pragma unroll
        for (int j = 0; j < 16; ++j) al[j] = s;
    } else if (GATE == KDA_GATE_NONE) {
#pragma unroll
        for (int j = 0; j < 16; ++j) al[j] = 1.0f;
    }
    float kq = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        qr[j] *= a.scale;
        kq = fmaf(kr[j], qr[j], kq);
    }
    kq += __shfl_xor_sync(0xffffffffu, kq, 1);
    kq += __shfl_xor_sync(0xffffffffu, kq, 2);
    kq += __shfl_xor_sync(0xffffffffu, kq, 4);
    const float beta = __ldg(a.beta + nh);

    const int row0 = blockIdx.y * kRowsPerCta + warp * kRowsPerWarp + rsel;
    float* Sbase = a.S + (size_t)nh * a.d_v * kDK;
    const TI* vp = static_cast<const TI*>(a.v) + (size_t)nh * a.d_v;
    TI* op = static_cast<TI*>(a.out) + (size_t)nh * a.d_v;

    float s[4][16];
    float vr[4];
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int r = row0 + 4 * it;
        if (r < a.d_v) {
            const float* rowp = Sbase + (size_t)r * kDK + 4 * sub;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 t = __ldcs(reinterpret_cast<const float4*>(rowp + 32 * m));
                s[it][4 * m + 0] = t.x; s[it][4 * m + 1] = t.y;
                s[it][4 * m + 2] = t.z; s[it][4 * m + 3] = t.w;
            }
            vr[it] = to_f32(vp[r]);
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) s[it][j] = 0.f;
            vr[it] = 0.f;
        }
    }
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int r = row0 + 4 * it;
        float pa = 0.f, pb = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            s[it][j] *= al[j];
            pa = fmaf(s[it][j], kr[j], pa);
            pb = fmaf(s[it][j], qr[j], pb);
        }
        pa += __shfl_xor_sync(0xffffffffu, pa, 1);
        pb += __shfl_xor_sync(0xffffffffu, pb, 1);
        pa += __shfl_xor_sync(0xffffffffu, pa, 2);
        pb += __shfl_xor_sync(0xffffffffu, pb, 2);
        pa += __shfl_xor_sync(0xffffffffu, pa, 4);
        pb += __shfl_xor_sync(0xffffffffu, pb, 4);
        if (r < a.d_v) {
            const float e = beta * (vr[it] - pa);
            float* rowp = Sbase + (size_t)r * kDK + 4 * sub;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                float4 t;
                t.x = fmaf(e, kr[4 * m + 0], s[it][4 * m + 0]);
                t.y = fmaf(e, kr[4 * m + 1], s[it][4 * m + 1]);
                t.z = fmaf(e, kr[4 * m + 2], s[it][4 * m + 2]);
                t.w = fmaf(e, kr[4 * m + 3], s[it][4 * m + 3]);
                __stcs(reinterpret_cast<float4*>(rowp + 32 * m), t);
            }
            if (sub == 0) op[r] = from_f32<TI>(fmaf(e, kq, pb));
        }
    }
}

template <typename TI>
cudaError_t launch_typed(const DecodeArgs& a, cudaStream_t s) {
    const dim3 grid((unsigned)(a.N * a.H), (unsigned)((a.d_v + kRowsPerCta - 1) / kRowsPerCta));
    switch (a.gate) {
        case KDA_GATE_CHANNEL: kda_decode_kernel<TI, KDA_GATE_CHANNEL><<<grid, kThreads, 0, s>>>(a); break;
        case KDA_GATE_SCALAR: kda_decode_kernel<TI, KDA_GATE_SCALAR><<<grid, kThreads, 0, s>>>(a); break;
        default: kda_decode_kernel<TI, KDA_GATE_NONE><<<grid, kThreads, 0, s>>>(a); break;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, bool bf16, cudaStream_t s) {
    return bf16 ? launch_typed<__nv_bfloat16>(a, s) : launch_typed<float>(a, s);
}

}  // namespace kda
