// kda_recurrent_bwd.cu -- gradients of the KDA token loop (training), on CUDA
// cores.
//
// Forward, per token t and value head (the five-step update at the top of "You
// could have come up with Kimi Delta Attention"):
//     S~ = S_{t-1} Diag(alpha_t);  vh = S~ k;  e = beta (v - vh);  S_t = S~ + e k^T;
//     o_t = S_t q~,  q~ = d_k^{-1/2} q,  alpha = exp(g).
// Backward, walking the tokens in reverse with G = dL/dS_t (starting from
// dL/dS_T), for the loss sum(o * d_out) + sum(S_T * d_ST):
//     G += d_out_t q~^T;            dq~ = S_t^T d_out_t
//     de = G k;  dk = G^T e;  dbeta = (v - vh) . de;  dv = beta de
//     G += (-beta de) k^T;          dk += S~^T (-beta de)
//     dg = (column sums of S~ .* G) (times 1 for a scalar gate summed over channels)
//     G <- G Diag(alpha)            (now dL/dS_{t-1}; after the first token it is dL/dS0)
// Every state row evolves on its own given the token vectors, so a CTA owns 16
// rows of one (sequence, value head) state (one row per 8-lane group, lane =
// 16 key channels, as in the decode kernel) and the cross-row sums (dq, dk, dg,
// dbeta) are reduced in shared memory, then added to the fp32 outputs with
// atomics (several row blocks, and the value heads of a group, share them).
//
// S_{t-1} is needed in reverse order, so the kernel first runs the forward for
// its rows and stores the state every kSeg tokens (workspace), then, segment by
// segment from the end, walks the segment backwards in windows of kWin tokens:
// for each window (last first) it reloads the segment's starting state,
// recomputes the forward up to the window's end keeping S~_t of the window's
// tokens in shared memory, and walks those tokens backwards.  Windows shorter
// than the segment trade some recomputation for shared memory, i.e. for more
// resident warps.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kDK = 128;
constexpr int kRows = 16;              // state rows per CTA
constexpr int kThreads = 8 * kRows;    // one 8-lane group per row
constexpr int kSeg = 8;                // tokens per checkpoint segment

// kWin: tokens whose S~ is kept at once -- the whole segment (8) when the grid is
// small, half of it (4, one more resident CTA per SM) when the grid is large.
template <int kWin>
struct Smem {
    float al[kSeg][kDK], kk[kSeg][kDK], qs[kSeg][kDK];   // the segment's token vectors
    float sb[kWin][kRows][kDK];                          // S~_t of this CTA's rows (one window)
    float vr[kSeg][kRows], dor[kSeg][kRows], vh[kSeg][kRows];
    float beta[kSeg];
    float red[3][kRows][kDK];                            // per-row partials of dq~, dk, dg
    float redb[kRows];
};

template <typename TI, int GATE, int kWin>
__global__ void __launch_bounds__(kThreads, 1) kda_recurrent_bwd_kernel(RecurrentBwdArgs a) {
    extern __shared__ float4 smem_raw[];
    Smem<kWin>& sm = *reinterpret_cast<Smem<kWin>*>(smem_raw);
    const int nh = blockIdx.x;
    const int n = nh / a.H, h = nh - n * a.H;
    const int hk = h / (a.H / a.Hk);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int sub = lane & 7, rl = warp * 4 + (lane >> 3);   // local row 0..15
    const int rbase = blockIdx.y * kRows;
    const int row = rbase + rl;
    const bool live = row < a.d_v;
    const int T = a.T;
    const int nseg = (T + kSeg - 1) / kSeg;
    const TI* q = static_cast<const TI*>(a.q);
    const TI* k = static_cast<const TI*>(a.k);
    const TI* v = static_cast<const TI*>(a.v);
    const TI* dout = static_cast<const TI*>(a.d_out);
    // checkpoint c of this CTA's rows: the state before token c * kSeg
    float* ck = a.ws + ((size_t)nh * nseg * a.d_v + rbase) * kDK;
    auto ck_at = [&](int c) { return ck + (size_t)c * a.d_v * kDK; };

    // Token t of the segment into slot j: channels by thread (tid < 128 = kDK), rows by tid < 16.
    auto stage = [&](int t, int j) {
        const size_t tv = ((size_t)n * T + t) * a.H + h, tkk = ((size_t)n * T + t) * a.Hk + hk;
        float gc = 0.f;
        if (GATE == KDA_GATE_CHANNEL) gc = a.g[tv * kDK + tid];
        else if (GATE == KDA_GATE_SCALAR) gc = a.g[tv];
        sm.al[j][tid] = (GATE == KDA_GATE_NONE) ? 1.f : expf(gc);
        sm.kk[j][tid] = to_f32(k[tkk * kDK + tid]);
        sm.qs[j][tid] = to_f32(q[tkk * kDK + tid]) * a.scale;
        if (tid < kRows) {
            const int r = rbase + tid;
            sm.vr[j][tid] = r < a.d_v ? to_f32(v[tv * a.d_v + r]) : 0.f;
            sm.dor[j][tid] = r < a.d_v ? to_f32(dout[tv * a.d_v + r]) : 0.f;
        }
        if (tid == 0) sm.beta[j] = a.beta[tv];
    };
    // channels of this lane: c = 32 m + 4 sub + i
    auto ch = [&](int m, int i) { return 32 * m + 4 * sub + i; };
    auto rowsum8 = [&](float x) {
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        return x;
    };
    // one forward token from slot j: S <- S~ + e k^T; keeps S~ (window slot w) and vh when w >= 0
    auto fwd_token = [&](float (&S)[16], int j, int w) {
        const bool keep = w >= 0;
        float pa = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                S[4 * m + i] *= sm.al[j][ch(m, i)];
                pa = fmaf(S[4 * m + i], sm.kk[j][ch(m, i)], pa);
            }
        pa = rowsum8(pa);
        if (keep) {
#pragma unroll
            for (int m = 0; m < 4; ++m)
                *reinterpret_cast<float4*>(&sm.sb[w][rl][ch(m, 0)]) =
                    make_float4(S[4 * m], S[4 * m + 1], S[4 * m + 2], S[4 * m + 3]);
            if (sub == 0) sm.vh[j][rl] = pa;
        }
        const float e = sm.beta[j] * (sm.vr[j][rl] - pa);
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i) S[4 * m + i] = fmaf(e, sm.kk[j][ch(m, i)], S[4 * m + i]);
    };
    auto load_rows = [&](float (&X)[16], const float* src) {   // src: row-major [rows][kDK]
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
            if (live && src) t = *reinterpret_cast<const float4*>(src + (size_t)rl * kDK + ch(m, 0));
            X[4 * m] = t.x; X[4 * m + 1] = t.y; X[4 * m + 2] = t.z; X[4 * m + 3] = t.w;
        }
    };
    auto store_rows = [&](float* dst, const float (&X)[16]) {
        if (!live) return;
#pragma unroll
        for (int m = 0; m < 4; ++m)
            *reinterpret_cast<float4*>(dst + (size_t)rl * kDK + ch(m, 0)) =
                make_float4(X[4 * m], X[4 * m + 1], X[4 * m + 2], X[4 * m + 3]);
    };

    // ---- forward over every token, storing the state at each segment start
    float S[16];
    const size_t sg = (size_t)nh * a.d_v * kDK + (size_t)rbase * kDK;
    load_rows(S, a.S0 ? a.S0 + sg : nullptr);
    for (int s = 0; s < nseg; ++s) {
        store_rows(ck_at(s), S);
        const int t0 = s * kSeg, len = min(kSeg, T - t0);
        __syncthreads();   // the previous segment's slots are read
        for (int j = 0; j < len; ++j) stage(t0 + j, j);
        __syncthreads();
        for (int j = 0; j < len; ++j) fwd_token(S, j, -1);
    }

    // ---- backward, segment by segment from the end
    float G[16];
    load_rows(G, a.d_ST ? a.d_ST + sg : nullptr);
    for (int s = nseg - 1; s >= 0; --s) {
        const int t0 = s * kSeg, len = min(kSeg, T - t0);
        __syncthreads();
        for (int j = 0; j < len; ++j) stage(t0 + j, j);
        __syncthreads();
        for (int w0 = ((len - 1) / kWin) * kWin; w0 >= 0; w0 -= kWin) {
        const int w1 = min(w0 + kWin, len);
        load_rows(S, ck_at(s));   // this thread's own rows: written by it in the forward
        for (int j = 0; j < w1; ++j) fwd_token(S, j, j >= w0 ? j - w0 : -1);
        __syncthreads();
        for (int j = w1 - 1; j >= w0; --j) {
            const int t = t0 + j;
            const float b = sm.beta[j], vhv = sm.vh[j][rl], dov = sm.dor[j][rl];
            const float e = b * (sm.vr[j][rl] - vhv);
            float sb[16], pq[16];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 x = *reinterpret_cast<const float4*>(&sm.sb[j - w0][rl][ch(m, 0)]);
                sb[4 * m] = x.x; sb[4 * m + 1] = x.y; sb[4 * m + 2] = x.z; sb[4 * m + 3] = x.w;
            }
            // o_t = S_t q~:  G += d_out q~^T,  dq~ += S_t^T d_out
            float de = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int c = ch(i >> 2, i & 3);
                const float kc = sm.kk[j][c];
                pq[i] = (sb[i] + e * kc) * dov;
                G[i] = fmaf(dov, sm.qs[j][c], G[i]);
                de = fmaf(G[i], kc, de);
            }
            de = rowsum8(de);
            // S_t = S~ + e k^T, e = beta (v - S~ k)
            const float dvh = -b * de;
            float pk[16], pg[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int c = ch(i >> 2, i & 3);
                const float kc = sm.kk[j][c];
                pk[i] = G[i] * e + sb[i] * dvh;
                G[i] = fmaf(dvh, kc, G[i]);       // dS~
                pg[i] = sb[i] * G[i];              // dg: alpha dalpha = S~ .* dS~, summed over rows
                G[i] *= sm.al[j][c];               // dS_{t-1}
            }
            const size_t tv = ((size_t)n * T + t) * a.H + h;
            if (live && sub == 0) a.dv[tv * a.d_v + row] = b * de;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int c = ch(m, 0);
                *reinterpret_cast<float4*>(&sm.red[0][rl][c]) =
                    make_float4(pq[4 * m], pq[4 * m + 1], pq[4 * m + 2], pq[4 * m + 3]);
                *reinterpret_cast<float4*>(&sm.red[1][rl][c]) =
                    make_float4(pk[4 * m], pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]);
                *reinterpret_cast<float4*>(&sm.red[2][rl][c]) =
                    make_float4(pg[4 * m], pg[4 * m + 1], pg[4 * m + 2], pg[4 * m + 3]);
            }
            if (sub == 0) sm.redb[rl] = live ? (sm.vr[j][rl] - vhv) * de : 0.f;
            __syncthreads();
            {
                // thread tid = channel: sum the 16 rows, add to the outputs
                float sq = 0.f, sk = 0.f, sgc = 0.f;
#pragma unroll
                for (int r = 0; r < kRows; ++r) {
                    sq += sm.red[0][r][tid];
                    sk += sm.red[1][r][tid];
                    sgc += sm.red[2][r][tid];
                }
                const size_t tkk = ((size_t)n * T + t) * a.Hk + hk;
                atomicAdd(a.dq + tkk * kDK + tid, sq * a.scale);
                atomicAdd(a.dk + tkk * kDK + tid, sk);
                if (GATE == KDA_GATE_CHANNEL) {
                    atomicAdd(a.dg + tv * kDK + tid, sgc);
                } else if (GATE == KDA_GATE_SCALAR) {
                    float x = sgc;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                    if (lane == 0) atomicAdd(a.dg + tv, x);
                }
                if (tid == 0) {
                    float sb2 = 0.f;
#pragma unroll
                    for (int r = 0; r < kRows; ++r) sb2 += sm.redb[r];
                    atomicAdd(a.dbeta + tv, sb2);
                }
            }
            __syncthreads();   // red (and, after the window, sb) is rewritten next
        }
        }
    }
    if (a.dS0) store_rows(a.dS0 + sg, G);
}

template <typename TI, int GATE, int kWin>
cudaError_t launch_one(const RecurrentBwdArgs& a, dim3 grid, cudaStream_t st) {
    auto kern = kda_recurrent_bwd_kernel<TI, GATE, kWin>;
    const size_t bytes = sizeof(Smem<kWin>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, bytes, st>>>(a);
    return cudaGetLastError();
}

template <typename TI, int GATE>
cudaError_t launch_gate(const RecurrentBwdArgs& a, cudaStream_t st) {
    const dim3 grid((unsigned)(a.N * a.H), (unsigned)((a.d_v + kRows - 1) / kRows));
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    // many CTAs: residency pays more than the recomputation the half window costs
    const bool wide = (long long)grid.x * grid.y >= 8LL * sms;
    return wide ? launch_one<TI, GATE, kSeg / 2>(a, grid, st) : launch_one<TI, GATE, kSeg>(a, grid, st);
}

template <typename TI>
cudaError_t launch_typed(const RecurrentBwdArgs& a, cudaStream_t st) {
    switch (a.gate) {
        case KDA_GATE_CHANNEL: return launch_gate<TI, KDA_GATE_CHANNEL>(a, st);
        case KDA_GATE_SCALAR: return launch_gate<TI, KDA_GATE_SCALAR>(a, st);
        default: return launch_gate<TI, KDA_GATE_NONE>(a, st);
    }
}

}  // namespace

size_t recurrent_bwd_workspace_bytes(int N, int T, int H, int d_v) {
    const size_t nseg = ((size_t)T + kSeg - 1) / kSeg;
    return (size_t)N * H * nseg * d_v * kDK * sizeof(float);
}

cudaError_t launch_recurrent_bwd(const RecurrentBwdArgs& a, bool bf16, cudaStream_t st) {
    return bf16 ? launch_typed<__nv_bfloat16>(a, st) : launch_typed<float>(a, st);
}

}  // namespace kda
