// kda_recurrent.cu -- fused recurrent KDA over a short run of tokens per
// sequence (speculative / short prefill, stateful serving): the token loop of
// the five-step update at the top of "You could have come up with Kimi Delta
// Attention", kept in registers across the tokens, so the d_v x d_k state is
// read from HBM once and written once per call instead of once per token.
// It is the multi-token form of the fused recurrent decode schedule (GeekNews
// summary, section "fused recurrent kernel for decode").
//
// Every state row r (value index) evolves independently given the token
// vectors, so the work layout follows the decode kernel's: a CTA owns 32 rows
// of one (n, h) state, each warp 4 rows, one row per 8-lane group (few
// registers, so two CTAs share an SM and hide each other's latency); lane
// (l & 7) holds key columns 4(l & 7) + 32m, m = 0..3.  Per token:
//     sd = S_r Diag(alpha_t); a = sd.k_t; b = sd.q~_t; e = beta_t (v_tr - a)
//     S_r <- sd + e k_t;      o_tr = b + e (k_t . q~_t)
// The next token's vectors are loaded while the current one is processed.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kDK = 128;           // key head size handled by this kernel
constexpr int kThreads = 256;      // 8 warps
constexpr int kIt = 1;             // rows per 8-lane group
constexpr int kRowsPerCta = 8 * 4 * kIt;

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

// One token's operands as this lane sees them.
template <typename TI>
struct TokenRegs {
    float k[16], q[16], g[16], v[kIt];
    float beta;
};

template <typename TI, int GATE>
__device__ __forceinline__ void load_token(const RecurrentArgs& a, size_t tok_h, const int* rows, int sub,
                                           TokenRegs<TI>& t) {
    const TI* kp = static_cast<const TI*>(a.k) + tok_h * kDK;
    const TI* qp = static_cast<const TI*>(a.q) + tok_h * kDK;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int c = 32 * m + 4 * sub;
        load4(kp + c, t.k + 4 * m);
        load4(qp + c, t.q + 4 * m);
        if (GATE == KDA_GATE_CHANNEL) load4(a.g + tok_h * kDK + c, t.g + 4 * m);
    }
    if (GATE == KDA_GATE_SCALAR) {
        const float s = __ldg(a.g + tok_h);
#pragma unroll
        for (int j = 0; j < 16; ++j) t.g[j] = s;
    }
    t.beta = __ldg(a.beta + tok_h);
    const TI* vp = static_cast<const TI*>(a.v) + tok_h * a.d_v;
#pragma unroll
    for (int it = 0; it < kIt; ++it) t.v[it] = rows[it] < a.d_v ? to_f32(vp[rows[it]]) : 0.f;
}

template <typename TI, int GATE>
__global__ void __launch_bounds__(kThreads, 2) kda_recurrent_kernel(RecurrentArgs a) {
    const int nh = blockIdx.x;
    const int n = nh / a.H, h = nh - n * a.H;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane & 7, rsel = lane >> 3;
    int rows[kIt];
#pragma unroll
    for (int it = 0; it < kIt; ++it) rows[it] = blockIdx.y * kRowsPerCta + warp * (4 * kIt) + rsel + 4 * it;

    float* Sbase = a.S + (size_t)nh * a.d_v * kDK;
    float s[kIt][16];
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        if (rows[it] < a.d_v) {
            const float* rowp = Sbase + (size_t)rows[it] * kDK + 4 * sub;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 t = __ldcs(reinterpret_cast<const float4*>(rowp + 32 * m));
                s[it][4 * m + 0] = t.x; s[it][4 * m + 1] = t.y;
                s[it][4 * m + 2] = t.z; s[it][4 * m + 3] = t.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) s[it][j] = 0.f;
        }
    }

    TokenRegs<TI> cur, nxt;
    const size_t tok0 = (size_t)n * a.T;
    if (a.T > 0) load_token<TI, GATE>(a, tok0 * a.H + h, rows, sub, cur);
    TI* out = static_cast<TI*>(a.out);
    for (int t = 0; t < a.T; ++t) {
        if (t + 1 < a.T) load_token<TI, GATE>(a, (tok0 + t + 1) * a.H + h, rows, sub, nxt);
        float al[16], qs[16];
        float kq = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            al[j] = (GATE == KDA_GATE_NONE) ? 1.f : expf(cur.g[j]);
            qs[j] = cur.q[j] * a.scale;
            kq = fmaf(cur.k[j], qs[j], kq);
        }
        kq += __shfl_xor_sync(0xffffffffu, kq, 1);
        kq += __shfl_xor_sync(0xffffffffu, kq, 2);
        kq += __shfl_xor_sync(0xffffffffu, kq, 4);
        const size_t orow = ((tok0 + t) * a.H + h) * a.d_v;
#pragma unroll
        for (int it = 0; it < kIt; ++it) {
            float pa = 0.f, pb = 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                s[it][j] *= al[j];
                pa = fmaf(s[it][j], cur.k[j], pa);
                pb = fmaf(s[it][j], qs[j], pb);
            }
            pa += __shfl_xor_sync(0xffffffffu, pa, 1);
            pb += __shfl_xor_sync(0xffffffffu, pb, 1);
            pa += __shfl_xor_sync(0xffffffffu, pa, 2);
            pb += __shfl_xor_sync(0xffffffffu, pb, 2);
            pa += __shfl_xor_sync(0xffffffffu, pa, 4);
            pb += __shfl_xor_sync(0xffffffffu, pb, 4);
            const float e = cur.beta * (cur.v[it] - pa);
#pragma unroll
            for (int j = 0; j < 16; ++j) s[it][j] = fmaf(e, cur.k[j], s[it][j]);
            if (sub == 0 && rows[it] < a.d_v) out[orow + rows[it]] = from_f32<TI>(fmaf(e, kq, pb));
        }
        cur = nxt;
    }

#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        if (rows[it] < a.d_v) {
            float* rowp = Sbase + (size_t)rows[it] * kDK + 4 * sub;
#pragma unroll
            for (int m = 0; m < 4; ++m)
                __stcs(reinterpret_cast<float4*>(rowp + 32 * m),
                       make_float4(s[it][4 * m], s[it][4 * m + 1], s[it][4 * m + 2], s[it][4 * m + 3]));
        }
    }
}

template <typename TI>
cudaError_t launch_typed(const RecurrentArgs& a, cudaStream_t st) {
    const dim3 grid((unsigned)(a.N * a.H), (unsigned)((a.d_v + kRowsPerCta - 1) / kRowsPerCta));
    switch (a.gate) {
        case KDA_GATE_CHANNEL: kda_recurrent_kernel<TI, KDA_GATE_CHANNEL><<<grid, kThreads, 0, st>>>(a); break;
        case KDA_GATE_SCALAR: kda_recurrent_kernel<TI, KDA_GATE_SCALAR><<<grid, kThreads, 0, st>>>(a); break;
        default: kda_recurrent_kernel<TI, KDA_GATE_NONE><<<grid, kThreads, 0, st>>>(a); break;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_recurrent(const RecurrentArgs& a, bool bf16, cudaStream_t st) {
    return bf16 ? launch_typed<__nv_bfloat16>(a, st) : launch_typed<float>(a, st);
}

}  // namespace kda
