// kda_chunk_bwd_grad.cu -- the chunk-parallel half of the chunkwise backward.
//
// With every chunk's incoming state S (checkpointed by the forward scan), the
// gradient of its outgoing state dS' and dE^T (both from the reverse scan), the
// gradients of a chunk's inputs depend on that chunk alone, so one CTA per
// (chunk, head) forms them.  The chunk map is the forward's (the GeekNews summary
// of "You could have come up with Kimi Delta Attention", section "Chunkwise KDA";
// the triangular solve the curriculum page names):
//
//   Gamma = cumsum(g),  A_ij = sum_c K_ic K_jc e^{Gamma_ic - Gamma_jc} (j < i),
//   M = I + strict_lower(diag(beta) A),  resid = V - (K e^Gamma) S^T,
//   E = M^{-1} diag(beta) resid,  Aqk_ij = sum_c Q~_ic K_jc e^{Gamma_ic - Gamma_jc} (j <= i),
//   O = (Q~ e^Gamma) S^T + Aqk E,  S' = S Diag(e^gamma) + E^T (K e^{gamma - Gamma}),
//
// and the gradients below are its chain rule, step by step in reverse (the pages
// give no backward derivation):
//
//   solve kernel (one CTA per (chunk, head)):
//     dEbar = M^{-T} dE (back substitution),  dbeta = rowsum(dEbar . resid) + rowsum(dL . A),
//     dL = strict_lower(-dEbar E^T),  dv = diag(beta) dEbar,
//     and for the next kernel E^T, dPr^T = -(diag(beta) dEbar)^T and dA = diag(beta) dL;
//   dqk kernel:
//     dKd = E dS',  dQg = dO S,  dKg = dPr S  (one fused pass over the state rows),
//     dAqk = lower(dO E^T), the two decay-weighted Gram products' own gradients,
//     dgamma = colsum(S . dS') e^gamma + colsum(dKd . Kd), dg = reverse cumsum of dGamma.
//
// The decay factor e^{Gamma_ic - Gamma_jc} of a Gram entry is split over 16-token
// sub-blocks I (of i) and J (of j), with r(I) the sub-block's first row:
//   a_ic = 2^{G_ic - G_r(I)c} <= 1,  b_jc = 2^{G_r(J)c - G_jc} (its own sub-block only),
//   d^{IJ}_c = 2^{G_r(I)c - G_r(J)c} <= 1 (J < I),   (G = Gamma in log2 units)
// so every Gram product and its gradient becomes a plain product of row-scaled
// operands with a per-column factor per sub-block pair; b stays bounded by the decay
// of 15 tokens.  Everything here is fp32 on CUDA cores.
#include <cuda_bf16.h>

#include "kda_chunk_bwd.cuh"
#include "kda_tc_common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace tc;
using sm100::pdl_wait;

constexpr int C = rec::C, DK = rec::DK, DV = rec::DV, NT = 256;
constexpr int LD = 132;          // fp32 row stride of [64][128] tiles
constexpr int LT = 68;           // fp32 row stride of [128][64] and [64][64] tiles
constexpr int REG = 128 * LT;    // floats per shared-memory region
static_assert(REG >= 64 * LD, "a region holds either tile shape");
constexpr float kLog2e = 1.4426950408889634f;

constexpr int SOLVE_FLOATS = 5 * REG + C * LT + 6 * DK + C;
constexpr int DQK_FLOATS = 4 * REG + 2 * C * LT + 2 * C * LT + 6 * DK + 16 * C;
constexpr int SOLVE_SMEM = SOLVE_FLOATS * 4;
constexpr int DQK_SMEM = DQK_FLOATS * 4;
static_assert(SOLVE_SMEM <= 232448 && DQK_SMEM <= 232448, "shared memory over the sm_100 per-block limit");

struct GradParams {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    const __nv_bfloat16* d_out;
    const float* g;
    const float* beta;
    const int32_t* cu_seqlens;
    const int32_t* coff;
    const float* chk;     // [slot][H][d_v][d_k]
    const float* dsp;     // [slot][H][d_v][d_k]
    float* de;            // [slot][H][d_v][C]: dE^T in, dPr^T out
    float* et;            // [slot][H][d_v][C]
    float* da;            // [slot][H][C][C]
    float* dq;
    float* dk;
    float* dv;
    float* dg;
    float* dbeta;
    int T, H, num_seqs, nc, group;
    float scale;
};

// Slot -> (first row c0, length L).  False for slots past the last chunk.
__device__ __forceinline__ bool slot_rows(const GradParams& p, int slot, long long& c0, int& L) {
    if (p.cu_seqlens == nullptr) {
        const int n = slot / p.nc, m = slot % p.nc;
        c0 = (long long)n * p.T + (long long)m * C;
        L = min(C, p.T - m * C);
        return L > 0;
    }
    if (slot >= p.coff[p.num_seqs]) return false;
    int lo = 0, hi = p.num_seqs - 1;   // largest n with coff[n] <= slot
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.coff[mid] <= slot) lo = mid; else hi = mid - 1;
    }
    const long long bos = p.cu_seqlens[lo], eos = p.cu_seqlens[lo + 1];
    c0 = bos + (long long)(slot - p.coff[lo]) * C;
    L = (int)min((long long)C, eos - c0);
    return L > 0;
}

__device__ __forceinline__ int pair_index(int I, int J) { return I * (I - 1) / 2 + J; }   // J < I

// G = cumulative log2 decay of the chunk (rows past L carry no decay), threads 0..127.
template <int GATE>
__device__ __forceinline__ void load_gamma(const GradParams& p, long long c0, int L, int h, float* sG) {
    const int c = threadIdx.x;
    if (c >= DK) return;
    float acc = 0.f;
#pragma unroll 8
    for (int i = 0; i < C; ++i) {
        float gv = 0.f;
        if (GATE == KDA_GATE_CHANNEL) {
            if (i < L) gv = p.g[((c0 + i) * p.H + h) * DK + c];
        } else if (GATE == KDA_GATE_SCALAR) {
            if (i < L) gv = p.g[(c0 + i) * p.H + h];
        }
        acc += gv * kLog2e;
        sG[i * LD + c] = acc;
    }
}

// d^{IJ}_c for the six sub-block pairs J < I.
__device__ __forceinline__ void load_dfac(const float* sG, float* dfac) {
    for (int x = threadIdx.x; x < 6 * DK; x += NT) {
        const int pi = x / DK, c = x % DK;
        const int I = pi < 1 ? 1 : (pi < 3 ? 2 : 3), J = pi - I * (I - 1) / 2;
        dfac[x] = ex2(sG[16 * I * LD + c] - sG[16 * J * LD + c]);
    }
}

// 8 bf16 values of row `row` (or zeros past the chunk).
__device__ __forceinline__ void load8(const __nv_bfloat16* base, bool valid, float* f) {
    if (valid) {
        unpack8(__ldg(reinterpret_cast<const uint4*>(base)), f);
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = 0.f;
    }
}

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void st4(float* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
__device__ __forceinline__ float comp(const float4& x, int e) {
    return e == 0 ? x.x : (e == 1 ? x.y : (e == 2 ? x.z : x.w));
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sm100::smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// ---------------------------------------------------------------- solve kernel
template <int GATE>
__global__ void __launch_bounds__(NT, 1) kda_chunk_bwd_solve_kernel(const __grid_constant__ GradParams p) {
    extern __shared__ float4 smem4[];
    float* sG = reinterpret_cast<float*>(smem4);   // [64][LD] G (log2 units)
    float* R1 = sG + REG;                          // K a  -> (K e^Gamma)^T [128][LT]
    float* R2 = R1 + REG;                          // K b  -> resid^T [128][LT]
    float* R3 = R2 + REG;                          // E^T [128][LT]
    float* R4 = R3 + REG;                          // dE^T -> dEbar^T [128][LT]
    float* sA = R4 + REG;                          // [64][LT] A, strictly lower
    float* dfac = sA + C * LT;                     // [6][128]
    float* sb = dfac + 6 * DK;                     // [64] beta
    float* red = R1;                               // after the resid product: dbeta partial sums
                                                   // [4 + 16][64], summed in a fixed order
    const int tid = threadIdx.x;
    const int slot = blockIdx.x / p.H, h = blockIdx.x % p.H, hk = h / p.group;
    pdl_wait();
    long long c0;
    int L;
    if (!slot_rows(p, slot, c0, L)) return;
    const size_t sh = (size_t)slot * p.H + h;

    load_gamma<GATE>(p, c0, L, h, sG);
    if (tid < C) sb[tid] = tid < L ? p.beta[(c0 + tid) * p.H + h] : 0.f;
    {
        const float4* src = reinterpret_cast<const float4*>(p.de + sh * DV * C);
        for (int x = tid; x < DV * C / 4; x += NT) *reinterpret_cast<float4*>(R4 + (x >> 4) * LT + 4 * (x & 15)) = src[x];
    }
    // this thread's K: rows i = x & 63, 8-channel chunk x >> 6, for x = tid + 256 r
    float kr[4][8];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int x = tid + NT * r, i = x & 63, cc = x >> 6;
        load8(p.k + ((c0 + i) * (p.H / p.group) + hk) * DK + 8 * cc, i < L, kr[r]);
    }
    __syncthreads();
    load_dfac(sG, dfac);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int x = tid + NT * r, i = x & 63, cc = x >> 6;
        const float* Gi = sG + i * LD + 8 * cc;
        const float* Gr = sG + (i & ~15) * LD + 8 * cc;
        float ka[8], kb[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            ka[e] = kr[r][e] * ex2(Gi[e] - Gr[e]);
            kb[e] = kr[r][e] * ex2(Gr[e] - Gi[e]);
        }
        st4(R1 + i * LD + 8 * cc, ka[0], ka[1], ka[2], ka[3]);
        st4(R1 + i * LD + 8 * cc + 4, ka[4], ka[5], ka[6], ka[7]);
        st4(R2 + i * LD + 8 * cc, kb[0], kb[1], kb[2], kb[3]);
        st4(R2 + i * LD + 8 * cc + 4, kb[4], kb[5], kb[6], kb[7]);
    }
    __syncthreads();

    // ---- A (strictly lower): tiles of 4 rows x 4 columns
    {
        const int ig = tid & 15, jg = tid >> 4, I = ig >> 2, J = jg >> 2;
        float acc[4][4] = {};
        if (J <= I) {
            const float* dv = dfac + (J < I ? pair_index(I, J) : 0) * DK;
            for (int c = 0; c < DK; c += 4) {
                float4 a[4], b[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    a[r] = ld4(R1 + (4 * ig + r) * LD + c);
                    b[r] = ld4(R2 + (4 * jg + r) * LD + c);
                }
                if (J < I) {
                    const float4 d = ld4(dv + c);
#pragma unroll
                    for (int r = 0; r < 4; ++r) b[r].x *= d.x, b[r].y *= d.y, b[r].z *= d.z, b[r].w *= d.w;
                }
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
                        acc[r][s] = fmaf(a[r].x, b[s].x, acc[r][s]);
                        acc[r][s] = fmaf(a[r].y, b[s].y, acc[r][s]);
                        acc[r][s] = fmaf(a[r].z, b[s].z, acc[r][s]);
                        acc[r][s] = fmaf(a[r].w, b[s].w, acc[r][s]);
                    }
            }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int i = 4 * ig + r;
            float o[4];
#pragma unroll
            for (int s = 0; s < 4; ++s) o[s] = (4 * jg + s < i) ? acc[r][s] : 0.f;
            st4(sA + i * LT + 4 * jg, o[0], o[1], o[2], o[3]);
        }
    }
    __syncthreads();
    // (K e^Gamma)^T into R1
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int x = tid + NT * r, i = x & 63, cc = x >> 6;
#pragma unroll
        for (int e = 0; e < 8; ++e) R1[(8 * cc + e) * LT + i] = kr[r][e] * ex2(sG[i * LD + 8 * cc + e]);
    }
    __syncthreads();

    // ---- resid^T = V^T - S (K e^Gamma)^T: rows v = 8 vg .. +7, columns i = 4 ig .. +3
    {
        const int vg = tid >> 4, ig = tid & 15;
        const float* S = p.chk + sh * DV * DK + (size_t)(8 * vg) * DK;
        float acc[8][4] = {};
        float4 cur[8], nxt[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) cur[r] = __ldg(reinterpret_cast<const float4*>(S + r * DK));
#pragma unroll 2
        for (int c = 0; c < DK; c += 4) {
            if (c + 4 < DK) {
#pragma unroll
                for (int r = 0; r < 8; ++r) nxt[r] = __ldg(reinterpret_cast<const float4*>(S + r * DK + c + 4));
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float4 kg = ld4(R1 + (c + e) * LT + 4 * ig);
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const float s = comp(cur[r], e);
                    acc[r][0] = fmaf(s, kg.x, acc[r][0]);
                    acc[r][1] = fmaf(s, kg.y, acc[r][1]);
                    acc[r][2] = fmaf(s, kg.z, acc[r][2]);
                    acc[r][3] = fmaf(s, kg.w, acc[r][3]);
                }
            }
#pragma unroll
            for (int r = 0; r < 8; ++r) cur[r] = nxt[r];
        }
        float vv[4][8];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int i = 4 * ig + s;
            load8(p.v + ((c0 + i) * p.H + h) * DV + 8 * vg, i < L, vv[s]);
        }
#pragma unroll
        for (int r = 0; r < 8; ++r)
            st4(R2 + (8 * vg + r) * LT + 4 * ig, vv[0][r] - acc[r][0], vv[1][r] - acc[r][1], vv[2][r] - acc[r][2],
                vv[3][r] - acc[r][3]);
    }
    __syncthreads();

    // ---- E = M^{-1} diag(beta) resid and dEbar = M^{-T} dE, per value row v: two
    // threads per row split every sum by the parity of its index (each keeps the
    // entries of its own parity) and meet through one shuffle.
    {
        const int v = tid >> 1, par = tid & 1;
        const float* rs = R2 + v * LT;
        float* er = R3 + v * LT;
        for (int i = 0; i < C; ++i) {
            float part = 0.f;
            for (int j = par; j < i; j += 2) part = fmaf(sA[i * LT + j], er[j], part);
            const float tot = part + __shfl_xor_sync(0xffffffffu, part, 1);
            if ((i & 1) == par) er[i] = sb[i] * (rs[i] - tot);
        }
        float* dr = R4 + v * LT;
        for (int j = C - 1; j >= 0; --j) {
            float part = 0.f;
            int i0 = j + 1;
            if ((i0 & 1) != par) ++i0;
            for (int i = i0; i < C; i += 2) part = fmaf(sb[i] * sA[i * LT + j], dr[i], part);
            const float tot = part + __shfl_xor_sync(0xffffffffu, part, 1);
            if ((j & 1) == par) dr[j] -= tot;
        }
    }
    __syncthreads();

    // ---- dbeta: rowsum(dEbar . resid) + rowsum(dL . A);  dL = -dEbar E^T, dA = diag(beta) dL
    {
        const int i = tid & 63, vq = tid >> 6;
        float s = 0.f;
        for (int v = 32 * vq; v < 32 * vq + 32; ++v) s = fmaf(R4[v * LT + i], R2[v * LT + i], s);
        red[vq * C + i] = s;
    }
    {
        const int ig = tid & 15, jg = tid >> 4;
        float acc[4][4] = {};
        if (jg <= ig) {
            for (int v = 0; v < DV; ++v) {
                const float4 a = ld4(R4 + v * LT + 4 * ig), e = ld4(R3 + v * LT + 4 * jg);
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const float ar = comp(a, r);
                    acc[r][0] = fmaf(ar, e.x, acc[r][0]);
                    acc[r][1] = fmaf(ar, e.y, acc[r][1]);
                    acc[r][2] = fmaf(ar, e.z, acc[r][2]);
                    acc[r][3] = fmaf(ar, e.w, acc[r][3]);
                }
            }
        }
        float* da = p.da + sh * C * C;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int i = 4 * ig + r;
            float o[4], dbp = 0.f;
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const int j = 4 * jg + s;
                const float dl = j < i ? -acc[r][s] : 0.f;
                dbp = fmaf(dl, sA[i * LT + j], dbp);
                o[s] = sb[i] * dl;
            }
            st4(da + i * C + 4 * jg, o[0], o[1], o[2], o[3]);
            red[(4 + jg) * C + i] = dbp;
        }
    }
    __syncthreads();

    if (tid < L) {
        float s = 0.f;
#pragma unroll
        for (int q = 0; q < 20; ++q) s += red[q * C + tid];
        p.dbeta[(c0 + tid) * p.H + h] = s;
    }
    {
        const int v = tid & 127;
        for (int i = tid >> 7; i < L; i += 2) p.dv[((c0 + i) * p.H + h) * DV + v] = sb[i] * R4[v * LT + i];
    }
    {
        float4* de = reinterpret_cast<float4*>(p.de + sh * DV * C);
        float4* et = reinterpret_cast<float4*>(p.et + sh * DV * C);
        for (int x = tid; x < DV * C / 4; x += NT) {
            const int v = x >> 4, i = 4 * (x & 15);
            const float4 d = ld4(R4 + v * LT + i);
            de[x] = make_float4(-sb[i] * d.x, -sb[i + 1] * d.y, -sb[i + 2] * d.z, -sb[i + 3] * d.w);
            et[x] = ld4(R3 + v * LT + i);
        }
    }
}

// ---------------------------------------------------------------- dqk kernel
template <int GATE>
__global__ void __launch_bounds__(NT, 1) kda_chunk_bwd_dqk_kernel(const __grid_constant__ GradParams p) {
    extern __shared__ float4 smem4[];
    float* sG = reinterpret_cast<float*>(smem4);   // [64][LD] G (log2 units)
    float* R1 = sG + REG;                          // E^T [128][LT]   -> K a [64][LD]
    float* R2 = R1 + REG;                          // dO^T [128][LT]  -> Q~ a
    float* R3 = R2 + REG;                          // dPr^T [128][LT] -> K b
    float* sAqk = R3 + REG;                        // [64][LT] dAqk (lower, diagonal included)
    float* sDA = sAqk + C * LT;                    // [64][LT] dA (strictly lower)
    float* R4 = sDA + C * LT;                      // state-row ring, then dAqk^T and dA^T
    float* dfac = R4 + 2 * C * LT;                 // [6][128]
    float* sred = dfac + 6 * DK;                   // [16][64] scalar-gate partial row sums
    const int tid = threadIdx.x;
    const int slot = blockIdx.x / p.H, h = blockIdx.x % p.H, hk = h / p.group, Hk = p.H / p.group;
    pdl_wait();
    long long c0;
    int L;
    if (!slot_rows(p, slot, c0, L)) return;
    const size_t sh = (size_t)slot * p.H + h;
    const float* S = p.chk + sh * DV * DK;
    const float* dS = p.dsp + sh * DV * DK;
    // ring of 3 stages, each 8 state rows of S then 8 of dS' (2048 floats)
    auto issue = [&](int b) {
        float* stg = R4 + (b % 3) * 2048;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int x = tid + NT * q, which = x >> 8, rr = (x >> 5) & 7, c4 = x & 31;
            const float* src = (which ? dS : S) + (size_t)(8 * b + rr) * DK + 4 * c4;
            cp_async16(stg + which * 1024 + rr * 128 + 4 * c4, src);
        }
        cp_async_commit();
    };
    issue(0);
    issue(1);

    load_gamma<GATE>(p, c0, L, h, sG);
    {
        const float4* e4 = reinterpret_cast<const float4*>(p.et + sh * DV * C);
        const float4* p4 = reinterpret_cast<const float4*>(p.de + sh * DV * C);
        for (int x = tid; x < DV * C / 4; x += NT) {
            const int off = (x >> 4) * LT + 4 * (x & 15);
            *reinterpret_cast<float4*>(R1 + off) = e4[x];
            *reinterpret_cast<float4*>(R3 + off) = p4[x];
        }
        const float4* a4 = reinterpret_cast<const float4*>(p.da + sh * C * C);
        for (int x = tid; x < C * C / 4; x += NT) *reinterpret_cast<float4*>(sDA + (x >> 4) * LT + 4 * (x & 15)) = a4[x];
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {   // dO^T
        const int x = tid + NT * r, i = x & 63, cc = x >> 6;
        float o[8];
        load8(p.d_out + ((c0 + i) * p.H + h) * DV + 8 * cc, i < L, o);
#pragma unroll
        for (int e = 0; e < 8; ++e) R2[(8 * cc + e) * LT + i] = o[e];
    }
    __syncthreads();
    load_dfac(sG, dfac);

    // ---- dAqk = lower(dO E^T), diagonal included
    {
        const int ig = tid & 15, jg = tid >> 4;
        float acc[4][4] = {};
        if (jg <= ig) {
            for (int v = 0; v < DV; ++v) {
                const float4 a = ld4(R2 + v * LT + 4 * ig), e = ld4(R1 + v * LT + 4 * jg);
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const float ar = comp(a, r);
                    acc[r][0] = fmaf(ar, e.x, acc[r][0]);
                    acc[r][1] = fmaf(ar, e.y, acc[r][1]);
                    acc[r][2] = fmaf(ar, e.z, acc[r][2]);
                    acc[r][3] = fmaf(ar, e.w, acc[r][3]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int i = 4 * ig + r;
            float o[4];
#pragma unroll
            for (int s = 0; s < 4; ++s) o[s] = (4 * jg + s <= i) ? acc[r][s] : 0.f;
            st4(sAqk + i * LT + 4 * jg, o[0], o[1], o[2], o[3]);
        }
    }

    // ---- one pass over the state rows v: dKd = E dS', dQg = dO S, dKg = dPr S and
    // colsum(S . dS'); thread: rows i = 4 ig .. +3, channels c = 8 cg .. +7
    const int cg = tid >> 4, ig = tid & 15, I = ig >> 2;
    float xk[4][8] = {}, xq[4][8] = {}, xg[4][8] = {}, dgs[8] = {};
    for (int b = 0; b < DV / 8; ++b) {
        cp_async_wait1();
        __syncthreads();
        if (b + 2 < DV / 8) issue(b + 2); else cp_async_commit();
        const float* stg = R4 + (b % 3) * 2048;
#pragma unroll 2
        for (int rr = 0; rr < 8; ++rr) {
            const int v = 8 * b + rr;
            const float4 e = ld4(R1 + v * LT + 4 * ig), o = ld4(R2 + v * LT + 4 * ig), pr = ld4(R3 + v * LT + 4 * ig);
            const float4 s0 = ld4(stg + rr * 128 + 8 * cg), s1 = ld4(stg + rr * 128 + 8 * cg + 4);
            const float4 d0 = ld4(stg + 1024 + rr * 128 + 8 * cg), d1 = ld4(stg + 1024 + rr * 128 + 8 * cg + 4);
            const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
            const float dv[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float er = comp(e, r), orr = comp(o, r), pp = comp(pr, r);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    xk[r][c] = fmaf(er, dv[c], xk[r][c]);
                    xq[r][c] = fmaf(orr, sv[c], xq[r][c]);
                    xg[r][c] = fmaf(pp, sv[c], xg[r][c]);
                }
            }
#pragma unroll
            for (int c = 0; c < 8; ++c) dgs[c] = fmaf(sv[c], dv[c], dgs[c]);
        }
    }
    cp_async_wait0();

    // ---- element-wise: xk <- dK, xq <- dQ, xg <- dGamma (so far); dgam per channel
    float gam[8], dgam[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) gam[c] = sG[(C - 1) * LD + 8 * cg + c];
    {
        float dgp[8] = {};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int i = 4 * ig + r;
            float kx[8], qx[8];
            load8(p.k + ((c0 + i) * Hk + hk) * DK + 8 * cg, i < L, kx);
            load8(p.q + ((c0 + i) * Hk + hk) * DK + 8 * cg, i < L, qx);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float G = sG[i * LD + 8 * cg + c];
                const float eG = ex2(G), eD = ex2(gam[c] - G);
                const float Kd = kx[c] * eD, Kg = kx[c] * eG, Qg = qx[c] * p.scale * eG;
                const float dKd = xk[r][c], dQg = xq[r][c], dKg = xg[r][c];
                dgp[c] = fmaf(dKd, Kd, dgp[c]);
                xk[r][c] = dKd * eD + dKg * eG;
                xq[r][c] = dQg * eG;
                xg[r][c] = -dKd * Kd + dQg * Qg + dKg * Kg;
            }
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            float x = dgp[c];
            x += __shfl_xor_sync(0xffffffffu, x, 1);
            x += __shfl_xor_sync(0xffffffffu, x, 2);
            x += __shfl_xor_sync(0xffffffffu, x, 4);
            x += __shfl_xor_sync(0xffffffffu, x, 8);
            dgam[c] = dgs[c] * ex2(gam[c]) + x;
        }
    }
    __syncthreads();   // E^T, dO^T, dPr^T and the ring are dead from here on

    // K a, Q~ a, K b; dAqk^T and dA^T
    float* dAT = R4;
    float* dDT = R4 + C * LT;
    for (int x = tid; x < C * 16; x += NT) {
        const int i = x >> 4, cc = x & 15;
        float kx[8], qx[8];
        load8(p.k + ((c0 + i) * Hk + hk) * DK + 8 * cc, i < L, kx);
        load8(p.q + ((c0 + i) * Hk + hk) * DK + 8 * cc, i < L, qx);
        const float* Gi = sG + i * LD + 8 * cc;
        const float* Gr = sG + (i & ~15) * LD + 8 * cc;
        float ka[8], qa[8], kb[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float a = ex2(Gi[e] - Gr[e]), bb = ex2(Gr[e] - Gi[e]);
            ka[e] = kx[e] * a;
            qa[e] = qx[e] * p.scale * a;
            kb[e] = kx[e] * bb;
        }
        float* o1 = R1 + i * LD + 8 * cc;
        float* o2 = R2 + i * LD + 8 * cc;
        float* o3 = R3 + i * LD + 8 * cc;
        st4(o1, ka[0], ka[1], ka[2], ka[3]);
        st4(o1 + 4, ka[4], ka[5], ka[6], ka[7]);
        st4(o2, qa[0], qa[1], qa[2], qa[3]);
        st4(o2 + 4, qa[4], qa[5], qa[6], qa[7]);
        st4(o3, kb[0], kb[1], kb[2], kb[3]);
        st4(o3 + 4, kb[4], kb[5], kb[6], kb[7]);
    }
    for (int x = tid; x < C * C; x += NT) {
        const int i = x & 63, j = x >> 6;
        dAT[j * LT + i] = sAqk[i * LT + j];
        dDT[j * LT + i] = sDA[i * LT + j];
    }
    __syncthreads();

    // ---- the Gram gradients, i side: dP1 = a . sum_J d^{IJ} (dAqk_{I,J} K b_J), dP2 likewise
    // with dA; dQ += dP1, dK += dP2, dGamma += Q~ . dP1 + K . dP2
    {
        float x1[4][8] = {}, x2[4][8] = {};
        for (int J = 0; J <= I; ++J) {
            float dv[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) dv[c] = J < I ? dfac[pair_index(I, J) * DK + 8 * cg + c] : 1.f;
            for (int j = 16 * J; j < 16 * J + 16; ++j) {
                const float4 aq = ld4(dAT + j * LT + 4 * ig), ad = ld4(dDT + j * LT + 4 * ig);
                const float4 b0 = ld4(R3 + j * LD + 8 * cg), b1 = ld4(R3 + j * LD + 8 * cg + 4);
                const float kb[8] = {b0.x * dv[0], b0.y * dv[1], b0.z * dv[2], b0.w * dv[3],
                                     b1.x * dv[4], b1.y * dv[5], b1.z * dv[6], b1.w * dv[7]};
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const float q1 = comp(aq, r), q2 = comp(ad, r);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        x1[r][c] = fmaf(q1, kb[c], x1[r][c]);
                        x2[r][c] = fmaf(q2, kb[c], x2[r][c]);
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int i = 4 * ig + r;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int cc = 8 * cg + c;
                const float a = ex2(sG[i * LD + cc] - sG[16 * I * LD + cc]);
                xq[r][c] = fmaf(a, x1[r][c], xq[r][c]);
                xk[r][c] = fmaf(a, x2[r][c], xk[r][c]);
                xg[r][c] += R2[i * LD + cc] * x1[r][c] + R1[i * LD + cc] * x2[r][c];
            }
        }
    }
    // ---- j side: Y = sum_{I' >= J} d^{I'J} (dAqk_{I',J}^T Q~a_I' + dA_{I',J}^T K a_I');
    // dK += b . Y, dGamma -= K b . Y   (this thread's rows are j, in sub-block J = I)
    {
        float y[4][8] = {};
        for (int Ip = I; Ip < 4; ++Ip) {
            float dv[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) dv[c] = Ip > I ? dfac[pair_index(Ip, I) * DK + 8 * cg + c] : 1.f;
            for (int i = 16 * Ip; i < 16 * Ip + 16; ++i) {
                const float4 aq = ld4(sAqk + i * LT + 4 * ig), ad = ld4(sDA + i * LT + 4 * ig);
                const float4 q0 = ld4(R2 + i * LD + 8 * cg), q1 = ld4(R2 + i * LD + 8 * cg + 4);
                const float4 k0 = ld4(R1 + i * LD + 8 * cg), k1 = ld4(R1 + i * LD + 8 * cg + 4);
                const float qa[8] = {q0.x * dv[0], q0.y * dv[1], q0.z * dv[2], q0.w * dv[3],
                                     q1.x * dv[4], q1.y * dv[5], q1.z * dv[6], q1.w * dv[7]};
                const float ka[8] = {k0.x * dv[0], k0.y * dv[1], k0.z * dv[2], k0.w * dv[3],
                                     k1.x * dv[4], k1.y * dv[5], k1.z * dv[6], k1.w * dv[7]};
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const float w1 = comp(aq, r), w2 = comp(ad, r);
#pragma unroll
                    for (int c = 0; c < 8; ++c) y[r][c] = fmaf(w1, qa[c], fmaf(w2, ka[c], y[r][c]));
                }
            }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int j = 4 * ig + r;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int cc = 8 * cg + c;
                const float b = ex2(sG[16 * I * LD + cc] - sG[j * LD + cc]);
                xk[r][c] = fmaf(b, y[r][c], xk[r][c]);
                xg[r][c] -= R3[j * LD + cc] * y[r][c];
            }
        }
    }

    // ---- dg = reverse cumulative sum of dGamma (gamma = Gamma of the last row)
    if (ig == 15) {
#pragma unroll
        for (int c = 0; c < 8; ++c) xg[3][c] += dgam[c];
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const float s3 = xg[3][c], s2 = xg[2][c] + s3, s1 = xg[1][c] + s2, s0 = xg[0][c] + s1;
        float incl = s0;
#pragma unroll
        for (int off = 1; off < 16; off <<= 1) {
            const float y = __shfl_down_sync(0xffffffffu, incl, off, 16);
            if (ig + off < 16) incl += y;
        }
        const float excl = incl - s0;
        xg[0][c] = s0 + excl;
        xg[1][c] = s1 + excl;
        xg[2][c] = s2 + excl;
        xg[3][c] = s3 + excl;
    }

    // ---- outputs
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int i = 4 * ig + r;
        if (i >= L) continue;
        const long long row = c0 + i;
        float* dq = p.dq + (row * Hk + hk) * DK + 8 * cg;
        float* dk = p.dk + (row * Hk + hk) * DK + 8 * cg;
        if (p.group == 1) {
            st4(dq, xq[r][0] * p.scale, xq[r][1] * p.scale, xq[r][2] * p.scale, xq[r][3] * p.scale);
            st4(dq + 4, xq[r][4] * p.scale, xq[r][5] * p.scale, xq[r][6] * p.scale, xq[r][7] * p.scale);
            st4(dk, xk[r][0], xk[r][1], xk[r][2], xk[r][3]);
            st4(dk + 4, xk[r][4], xk[r][5], xk[r][6], xk[r][7]);
        } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                atomicAdd(dq + c, xq[r][c] * p.scale);
                atomicAdd(dk + c, xk[r][c]);
            }
        }
        if (GATE == KDA_GATE_CHANNEL) {
            float* dg = p.dg + (row * p.H + h) * DK + 8 * cg;
            st4(dg, xg[r][0], xg[r][1], xg[r][2], xg[r][3]);
            st4(dg + 4, xg[r][4], xg[r][5], xg[r][6], xg[r][7]);
        } else if (GATE == KDA_GATE_SCALAR) {
            float s = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) s += xg[r][c];
            sred[cg * C + i] = s;
        }
    }
    if (GATE == KDA_GATE_SCALAR) {
        __syncthreads();
        if (tid < L) {
            float s = 0.f;
#pragma unroll
            for (int q = 0; q < 16; ++q) s += sred[q * C + tid];
            p.dg[(c0 + tid) * p.H + h] = s;
        }
    }
}

template <int GATE>
cudaError_t launch_grad_gate(const GradParams& p, unsigned grid, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(kda_chunk_bwd_solve_kernel<GATE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SOLVE_SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kda_chunk_bwd_dqk_kernel<GATE>, cudaFuncAttributeMaxDynamicSharedMemorySize, DQK_SMEM);
    if (e == cudaSuccess) e = launch_after(kda_chunk_bwd_solve_kernel<GATE>, dim3(grid), NT, SOLVE_SMEM, st, p);
    if (e == cudaSuccess) e = launch_after(kda_chunk_bwd_dqk_kernel<GATE>, dim3(grid), NT, DQK_SMEM, st, p);
    return e;
}

}  // namespace

cudaError_t launch_chunk_bwd_grad(const ChunkBwdArgs& a, uint8_t* ws, const BwdLayout& bl, cudaStream_t st) {
    GradParams p;
    p.q = static_cast<const __nv_bfloat16*>(a.q);
    p.k = static_cast<const __nv_bfloat16*>(a.k);
    p.v = static_cast<const __nv_bfloat16*>(a.v);
    p.d_out = static_cast<const __nv_bfloat16*>(a.d_out);
    p.g = a.g;
    p.beta = a.beta;
    p.cu_seqlens = a.cu_seqlens;
    p.coff = a.cu_seqlens ? reinterpret_cast<const int32_t*>(ws + bl.fwd.coff_off) : nullptr;
    p.chk = reinterpret_cast<const float*>(ws + bl.chk_off);
    p.dsp = reinterpret_cast<const float*>(ws + bl.dsp_off);
    p.de = reinterpret_cast<float*>(ws + bl.de_off);
    p.et = reinterpret_cast<float*>(ws + bl.et_off);
    p.da = reinterpret_cast<float*>(ws + bl.da_off);
    p.dq = a.dq;
    p.dk = a.dk;
    p.dv = a.dv;
    p.dg = a.dg;
    p.dbeta = a.dbeta;
    p.T = a.T;
    p.H = a.H;
    p.num_seqs = a.num_seqs;
    p.nc = (a.T + C - 1) / C;
    p.group = a.H / a.Hk;
    p.scale = a.scale;
    const long long grid = bl.fwd.slots * a.H;
    if (grid <= 0) return cudaSuccess;
    switch (a.gate) {
        case KDA_GATE_CHANNEL: return launch_grad_gate<KDA_GATE_CHANNEL>(p, (unsigned)grid, st);
        case KDA_GATE_SCALAR: return launch_grad_gate<KDA_GATE_SCALAR>(p, (unsigned)grid, st);
        default: return launch_grad_gate<KDA_GATE_NONE>(p, (unsigned)grid, st);
    }
}

}  // namespace kda
