// kda_chunk_f32.cu -- chunkwise KDA prefill on CUDA cores, fp32 arithmetic.
//
// This is the path for fp32 inputs and for head sizes the tensor-core path
// does not take (d_k, d_v multiples of 16 up to 128; chunk 16, 32 or 64).
// It follows the chunkwise form of the GeekNews summary of "You could have
// come up with Kimi Delta Attention" (section "Chunkwise KDA"), per chunk of
// C tokens with incoming state S_c (d_v x d_k):
//
//   Gamma_i = sum_{s<=i} g_s                        cumulative log decay (inclusive)
//   A_kk[i,j] = beta_i sum_c K_ic K_jc exp(Gamma_ic - Gamma_jc),  j < i   (coupling rho_ij)
//   A_qk[i,j] = sum_c Q~_ic K_jc exp(Gamma_ic - Gamma_jc),        j <= i
//   Ebar_i = beta_i (v_i - S_c (exp(Gamma_i) * k_i))    provisional errors
//   (I + A_kk) E = Ebar                                 forward substitution
//   o_i = S_c (exp(Gamma_i) * q~_i) + sum_{j<=i} A_qk[i,j] e_j
//   S_{c+1} = S_c Diag(exp(Gamma_last)) + sum_j e_j (k_j * exp(Gamma_last - Gamma_j))^T
//
// Every decay factor is exp of a difference of cumulative log gates taken
// with j <= i, so it never exceeds 1: the log-space ratios cannot overflow.
// One CTA per (sequence, head) walks its sequence's chunks in order with the
// state resident in shared memory (stored transposed, St[c][r], so the value
// index is the fast one for the state products).
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;

template <typename TI>
__device__ __forceinline__ float ld_in(const TI* p) { return to_f32(p[0]); }

struct Smem {
    float *K, *Q, *G, *E, *Akk, *Aqk, *St, *b, *glast;
};

__host__ __device__ inline size_t smem_floats(int C, int D, int V) {
    return (size_t)3 * C * D + (size_t)C * V + 2 * (size_t)C * C + (size_t)D * V + C + D;
}

template <typename TI, int GATE>
__global__ void __launch_bounds__(kThreads) kda_chunk_f32_kernel(ChunkArgs a) {
    extern __shared__ float4 smem_raw[];
    const int C = a.chunk, D = a.d_k, V = a.d_v, H = a.H;
    const int n = blockIdx.x / H, h = blockIdx.x % H;
    const int hk = h / (H / a.Hk);   // query/key head (grouped value heads share it)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    float* base = reinterpret_cast<float*>(smem_raw);
    Smem s;
    s.K = base;
    s.Q = s.K + C * D;
    s.G = s.Q + C * D;
    s.E = s.G + C * D;
    s.Akk = s.E + C * V;
    s.Aqk = s.Akk + C * C;
    s.St = s.Aqk + C * C;
    s.b = s.St + D * V;
    s.glast = s.b + C;

    long long bos, eos;
    if (!seq_bounds(a.cu_seqlens, n, a.T, a.num_seqs, a.dev_status, bos, eos)) return;

    const TI* q = static_cast<const TI*>(a.q);
    const TI* k = static_cast<const TI*>(a.k);
    const TI* v = static_cast<const TI*>(a.v);
    TI* out = static_cast<TI*>(a.out);

    // initial state, transposed into St[c][r]
    for (int idx = tid; idx < D * V; idx += kThreads) {
        const int r = idx / D, c = idx % D;
        s.St[c * V + r] = a.S0 ? a.S0[((size_t)n * H + h) * V * D + idx] : 0.f;
    }

    for (long long c0 = bos; c0 < eos; c0 += C) {
        const int L = (int)min((long long)C, eos - c0);
        __syncthreads();
        // ---- load the chunk (absent rows of a ragged chunk are zero: they
        //      neither couple nor write nor decay)
        for (int idx = tid; idx < C * D; idx += kThreads) {
            const int i = idx / D, c = idx % D;
            float kv = 0.f, qv = 0.f, gv = 0.f;
            if (i < L) {
                const size_t tok = (size_t)(c0 + i) * H + h, tk = (size_t)(c0 + i) * a.Hk + hk;
                kv = ld_in(k + tk * D + c);
                qv = ld_in(q + tk * D + c) * a.scale;
                if (GATE == KDA_GATE_CHANNEL) gv = a.g[tok * D + c];
                else if (GATE == KDA_GATE_SCALAR) gv = a.g[tok];
            }
            s.K[idx] = kv;
            s.Q[idx] = qv;
            s.G[idx] = gv;
        }
        for (int idx = tid; idx < C * V; idx += kThreads) {
            const int i = idx / V, r = idx % V;
            s.E[idx] = (i < L) ? ld_in(v + ((size_t)(c0 + i) * H + h) * V + r) : 0.f;
        }
        for (int i = tid; i < C; i += kThreads)
            s.b[i] = (i < L) ? a.beta[(size_t)(c0 + i) * H + h] : 0.f;
        __syncthreads();
        // ---- cumulative log decay, one thread per key channel
        for (int c = tid; c < D; c += kThreads) {
            float run = 0.f;
            for (int i = 0; i < C; ++i) {
                run += s.G[i * D + c];
                s.G[i * D + c] = run;
            }
            s.glast[c] = run;
        }
        __syncthreads();
        // ---- decay-masked key/key and query/key products; one warp per (i, j),
        //      lanes across key channels
        for (int i = warp; i < C; i += kThreads / 32) {
            for (int j = 0; j < C; ++j) {
                float skk = 0.f, sqk = 0.f;
                if (j <= i && i < L) {
                    for (int c = lane; c < D; c += 32) {
                        const float f = expf(s.G[i * D + c] - s.G[j * D + c]);
                        const float kj = s.K[j * D + c] * f;
                        skk = fmaf(s.K[i * D + c], kj, skk);
                        sqk = fmaf(s.Q[i * D + c], kj, sqk);
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        skk += __shfl_xor_sync(0xffffffffu, skk, o);
                        sqk += __shfl_xor_sync(0xffffffffu, sqk, o);
                    }
                }
                if (lane == 0) {
                    s.Akk[i * C + j] = (j < i) ? s.b[i] * skk : 0.f;
                    s.Aqk[i * C + j] = (j <= i) ? sqk : 0.f;
                }
            }
        }
        __syncthreads();
        // ---- fold the decay into the operands:
        //      G <- K exp(Gamma), K <- K exp(Gamma_last - Gamma), Q <- Q exp(Gamma)
        for (int idx = tid; idx < C * D; idx += kThreads) {
            const int c = idx % D;
            const float gam = s.G[idx];
            const float eg = expf(gam), ed = expf(s.glast[c] - gam);
            const float kv = s.K[idx];
            s.G[idx] = kv * eg;
            s.K[idx] = kv * ed;
            s.Q[idx] *= eg;
        }
        __syncthreads();
        // ---- provisional errors Ebar = diag(beta) (V - (K exp(Gamma)) S_c^T)
        for (int idx = tid; idx < C * V; idx += kThreads) {
            const int i = idx / V, r = idx % V;
            float acc = 0.f;
            for (int c = 0; c < D; ++c) acc = fmaf(s.G[i * D + c], s.St[c * V + r], acc);
            s.E[idx] = s.b[i] * (s.E[idx] - acc);
        }
        __syncthreads();
        // ---- (I + A_kk) E = Ebar by forward substitution; columns are independent
        for (int r = tid; r < V; r += kThreads) {
            for (int i = 1; i < L; ++i) {
                float acc = 0.f;
                for (int j = 0; j < i; ++j) acc = fmaf(s.Akk[i * C + j], s.E[j * V + r], acc);
                s.E[i * V + r] -= acc;
            }
        }
        __syncthreads();
        // ---- outputs o_i = S_c (exp(Gamma_i) q~_i) + sum_{j<=i} A_qk[i,j] e_j
        for (int idx = tid; idx < L * V; idx += kThreads) {
            const int i = idx / V, r = idx % V;
            float acc = 0.f;
            for (int c = 0; c < D; ++c) acc = fmaf(s.Q[i * D + c], s.St[c * V + r], acc);
            for (int j = 0; j <= i; ++j) acc = fmaf(s.Aqk[i * C + j], s.E[j * V + r], acc);
            out[((size_t)(c0 + i) * H + h) * V + r] = from_f32<TI>(acc);
        }
        __syncthreads();
        // ---- state: S_{c+1}^T = Diag(exp(Gamma_last)) S_c^T + (K exp(Gamma_last - Gamma))^T E
        for (int idx = tid; idx < D * V; idx += kThreads) {
            const int c = idx / V, r = idx % V;
            float acc = s.St[idx] * expf(s.glast[c]);
            for (int j = 0; j < L; ++j) acc = fmaf(s.K[j * D + c], s.E[j * V + r], acc);
            s.St[idx] = acc;
        }
    }
    __syncthreads();
    if (a.S_T) {
        for (int idx = tid; idx < D * V; idx += kThreads) {
            const int r = idx / D, c = idx % D;
            a.S_T[((size_t)n * H + h) * V * D + idx] = s.St[c * V + r];
        }
    }
}

template <typename TI, int GATE>
cudaError_t launch_gate(const ChunkArgs& a, cudaStream_t st) {
    const size_t bytes = smem_floats(a.chunk, a.d_k, a.d_v) * sizeof(float);
    auto kern = kda_chunk_f32_kernel<TI, GATE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(a.num_seqs * a.H), kThreads, bytes, st>>>(a);
    return cudaGetLastError();
}

template <typename TI>
cudaError_t launch_typed(const ChunkArgs& a, cudaStream_t st) {
    switch (a.gate) {
        case KDA_GATE_CHANNEL: return launch_gate<TI, KDA_GATE_CHANNEL>(a, st);
        case KDA_GATE_SCALAR: return launch_gate<TI, KDA_GATE_SCALAR>(a, st);
        default: return launch_gate<TI, KDA_GATE_NONE>(a, st);
    }
}

}  // namespace

size_t chunk_f32_smem_bytes(int C, int D, int V) { return smem_floats(C, D, V) * sizeof(float); }

cudaError_t launch_chunk_f32path(const ChunkArgs& a, bool bf16, cudaStream_t st) {
    return bf16 ? launch_typed<__nv_bfloat16>(a, st) : launch_typed<float>(a, st);
}

}  // namespace kda
