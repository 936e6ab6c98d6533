// kda_recurrent.cu -- fused recurrent KDA over a short run of tokens per
// sequence (speculative / short prefill, stateful serving): the token loop of
// the five-step update at the top of "You could have come up with Kimi Delta
// Attention", kept in registers across the tokens, so the d_v x d_k state is
// read from HBM once and written once per call instead of once per token.
// It is the multi-token form of the fused recurrent decode schedule (GeekNews
// summary, section "fused recurrent kernel for decode").
//
// Every state row r (value index) evolves independently given the token
// vectors, so the work layout follows the decode kernel's: a CTA owns 128
// rows of one (n, h) state, each warp 16, four at a time, one row per 8-lane
// group; lane (l & 7) holds key columns 4(l & 7) + 32m, m = 0..3.  Per token:
//     sd = S_r Diag(alpha_t); a = sd.k_t; b = sd.q~_t; e = beta_t (v_tr - a)
//     S_r <- sd + e k_t;      o_tr = b + e (k_t . q~_t)
// The token vectors alpha_t = exp(g_t), k_t, q~_t, beta_t and this CTA's
// entries of v_t are formed once per CTA in shared memory (double-buffered:
// the next token's are staged while the current one is processed); each lane
// reads its 16 channels of them.  The per-row arithmetic, including the
// k_t.q~_t partial sums, is the decode kernel's, operation for operation.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kDK = 128;           // key head size handled by this kernel
constexpr int kThreads = 256;      // 8 warps
constexpr int kIt = 4;             // rows per 8-lane group
constexpr int kRowsPerCta = 8 * 4 * kIt;
static_assert(kRowsPerCta == 128 && kThreads == 2 * kDK, "staging assigns one channel / row per thread");

struct Stage {
    float al[kDK], k[kDK], qs[kDK], v[kRowsPerCta];
    float beta, pad[3];
};

template <typename TI, int GATE>
__global__ void __launch_bounds__(kThreads, 2) kda_recurrent_kernel(RecurrentArgs a) {
    __shared__ __align__(16) Stage stg[2];
    const int nh = blockIdx.x;
    const int n = nh / a.H, h = nh - n * a.H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int sub = lane & 7, rsel = lane >> 3;
    const int rbase = blockIdx.y * kRowsPerCta;
    const int row0 = rbase + warp * (4 * kIt) + rsel;

    // Stage token t into buffer b: threads 0-127 own channel tid, 128-255 row tid - 128.
    const size_t tok0 = (size_t)n * a.T;
    const int hk = h / (a.H / a.Hk);   // query/key head (grouped value heads share it)
    auto stage = [&](int t, int b) {
        const size_t th = (tok0 + t) * a.H + h, tk = (tok0 + t) * a.Hk + hk;
        Stage& st = stg[b];
        if (tid < kDK) {
            float gc = 0.f;
            if (GATE == KDA_GATE_CHANNEL) gc = __ldg(a.g + th * kDK + tid);
            else if (GATE == KDA_GATE_SCALAR) gc = __ldg(a.g + th);
            st.al[tid] = (GATE == KDA_GATE_NONE) ? 1.f : expf(gc);
            st.k[tid] = to_f32(static_cast<const TI*>(a.k)[tk * kDK + tid]);
            st.qs[tid] = to_f32(static_cast<const TI*>(a.q)[tk * kDK + tid]) * a.scale;
            if (tid == 0) st.beta = __ldg(a.beta + th);
        } else {
            const int r = rbase + tid - kDK;
            st.v[tid - kDK] = r < a.d_v ? to_f32(static_cast<const TI*>(a.v)[th * a.d_v + r]) : 0.f;
        }
    };

    float* Sbase = a.S + (size_t)nh * a.d_v * kDK;
    float s[kIt][16];
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int r = row0 + 4 * it;
        if (r < a.d_v) {
            const float* rowp = Sbase + (size_t)r * kDK + 4 * sub;
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
    if (a.T > 0) stage(0, 0);
    __syncthreads();

    TI* out = static_cast<TI*>(a.out);
    for (int t = 0; t < a.T; ++t) {
        const int b = t & 1;
        if (t + 1 < a.T) stage(t + 1, b ^ 1);   // its loads overlap the work below
        const Stage& st = stg[b];
        float al[16], kr[16], qr[16];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int c = 32 * m + 4 * sub;
            const float4 x = *reinterpret_cast<const float4*>(st.al + c);
            const float4 y = *reinterpret_cast<const float4*>(st.k + c);
            const float4 z = *reinterpret_cast<const float4*>(st.qs + c);
            al[4 * m] = x.x; al[4 * m + 1] = x.y; al[4 * m + 2] = x.z; al[4 * m + 3] = x.w;
            kr[4 * m] = y.x; kr[4 * m + 1] = y.y; kr[4 * m + 2] = y.z; kr[4 * m + 3] = y.w;
            qr[4 * m] = z.x; qr[4 * m + 1] = z.y; qr[4 * m + 2] = z.z; qr[4 * m + 3] = z.w;
        }
        float kq = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) kq = fmaf(kr[j], qr[j], kq);
        kq += __shfl_xor_sync(0xffffffffu, kq, 1);
        kq += __shfl_xor_sync(0xffffffffu, kq, 2);
        kq += __shfl_xor_sync(0xffffffffu, kq, 4);
        const float beta = st.beta;
        const size_t orow = ((tok0 + t) * a.H + h) * a.d_v;
#pragma unroll
        for (int it = 0; it < kIt; ++it) {
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
            const float e = beta * (st.v[r - rbase] - pa);
#pragma unroll
            for (int j = 0; j < 16; ++j) s[it][j] = fmaf(e, kr[j], s[it][j]);
            if (sub == 0 && r < a.d_v) out[orow + r] = from_f32<TI>(fmaf(e, kq, pb));
        }
        __syncthreads();   // buffer b is re-staged next iteration; b ^ 1 is complete
    }

#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int r = row0 + 4 * it;
        if (r < a.d_v) {
            float* rowp = Sbase + (size_t)r * kDK + 4 * sub;
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
