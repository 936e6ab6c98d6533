// kda_chunk_tc.cu -- chunkwise KDA prefill on the sm_100a tensor cores
// (tcgen05 MMAs with fp32 accumulators in tensor memory, operands in shared
// memory, raw tiles brought in by TMA).  bf16 q/k/v, fp32 gates / beta /
// state, d_k = d_v = 128, chunk C = 64.
//
// The chunkwise form follows the GeekNews summary of "You could have come up
// with Kimi Delta Attention", section "Chunkwise KDA" (cumulative decay,
// provisional errors, coupling coefficients rho_ij), with the cut-off
// dependency formula completed as the unit-lower-triangular solve the
// curriculum page names ("pseudo-values from a triangular solve", "WY/UT
// form").  For a chunk of C tokens with incoming state S (d_v x d_k):
//
//   Gamma_i = sum_{s<=i} g_s                      (log-space cumulative decay)
//   P[i,j]  = sum_c K_ic K_jc e^{Gamma_ic - Gamma_jc}    (j <= i)
//   Qp[i,j] = sum_c Q~_ic K_jc e^{Gamma_ic - Gamma_jc}   (j <= i)
//   T       = (I + strict_lower(diag(beta) P))^{-1}
//   W = T diag(beta) (K e^{Gamma}),  U = T diag(beta) V  (pseudo-values)
//   E = U - W S^T                                     (true in-chunk errors)
//   O = (Q~ e^{Gamma}) S^T + lower(Qp) E              (outputs, post-write)
//   S^T <- Diag(e^{Gamma_last}) S^T + (K e^{Gamma_last - Gamma})^T E
//
// Log-space ratios.  A product e^{Gamma_i - Gamma_j} is split into two
// factors with a reference row r inside each 16-token sub-block:
// i-side x_i = e^{Gamma_i - Gamma_r(i)}, j-side e^{Gamma_r(I) - Gamma_j}; for
// j in an earlier sub-block the j-side factor is <= 1, and inside a sub-block
// both factors are bounded by e^{8 max|g|}, so nothing overflows in fp32/bf16
// for |g| up to ~10 per token.  e^{-Gamma} is never formed.
//
// Work layout: one CTA per (sequence, head, 64-wide value tile); the CTA walks
// its sequence's chunks in order with the fp32 state tile S^T (128 x 64) in
// registers (thread = key channel, half the value columns per warp group) and
// a bf16 copy in shared memory as the MMA operand.  The in-chunk phases run
// one after another; TMA for the next chunk is issued as soon as its landing
// buffers are free.
#include <cudaTypedefs.h>

#include "kda_internal.cuh"
#include "kda_tc_common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;
using namespace tc;

constexpr int C = 64, DK = 128, DV = 128, BV = 64, NVT = DV / BV, NT = 256;
constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s bound on every wait
// Issuing a tcgen05.mma holds the issuing thread while the tensor pipe takes it, so
// each batch is issued by a lane of a warp with no SIMT work in the phase that follows.
constexpr int kGramTid = 128;   // warp 4: only the dS / S update in finish_chunk
constexpr int kIssA = 192;      // warp 6: [-K e^G S^T ; O1], then O2
constexpr int kIssB = 224;      // warp 7: E, the next chunk's TMA, then dS

// Shared-memory map (bytes from a 1024-aligned base).
constexpr int OFF_RAW = 0;                       // raw K | raw Q | raw G  (64 KB)
constexpr int OFF_RK = OFF_RAW;                  //   [64][128] bf16
constexpr int OFF_RQ = OFF_RAW + 16384;          //   [64][128] bf16
constexpr int OFF_RG = OFF_RAW + 32768;          //   [64][128] fp32
constexpr int OFF_OX = OFF_RAW;                  // after prep (sub-block path): Gram B operand
constexpr int OFF_KYG = OFF_RAW;                 // after prep (one-reference path): K e^{-Gamma}
constexpr int OFF_KQG = OFF_RAW + 32768;         //   rows 0-63 K e^Gamma, rows 64-127 Q~ e^Gamma
// K e^{-Gamma}, the K|Q e^Gamma tile and K e^{Gamma_last - Gamma} share one layout,
// element (row n, channel c) at mnmaj_off(c, n, 128): 8-row groups 2048 bytes apart,
// 64-channel halves 1024 apart.  Read as MN-major (MN = c) or as K-major (K = c).
constexpr float kFastLimit2 = 112.f;             // one-reference path while max |Gamma_last| <= 2^112
constexpr int OFF_RV = 65536;                    // raw V tile, TMA 128B swizzle = MN-major operand
constexpr int OFF_A = 73728;                     // 64 KB, reused per phase:
constexpr int OFF_OY = OFF_A;                    //   Gram A operands: 2 K-major tiles of 128 rows
                                                 //   (tile g: rows 0-63 version 2g, 64-127 version 2g+1)
constexpr int OFF_TOT4 = OFF_A;                  //   decay scan (prep, before any operand write here):
constexpr int OFF_GREF = OFF_TOT4 + 8192;        //     fp32 [16][128] row-group sums then prefixes,
constexpr int OFF_GLAST = OFF_GREF + 2048;       //     [4][128] Gamma at reference rows, [128] at the
constexpr int OFF_RED = OFF_GLAST + 512;         //     last row, [4] per-warp max |Gamma_last| (log2)
constexpr int LDT = 68;                          //   fp32 row stride of L and T (bank spread)
constexpr int LDX = 20;                          //   fp32 row stride of 16x16 block scratch
constexpr int OFF_L = OFF_A;                     //   fp32 [64][LDT] coupling matrix L
constexpr int OFF_TF = OFF_L + 64 * LDT * 4;     //   fp32 [64][LDT] T = (I + L)^{-1}
constexpr int OFF_Q32 = OFF_TF + 64 * LDT * 4;   //   fp32 [64][LDT] lower(Qp), sub-block path
constexpr int OFF_NS = OFF_Q32 + 64 * LDT * 4;   //   fp32 [10][16][LDX] Neumann-series blocks
constexpr int OFF_TB = OFF_A + 65536;            // K-major, K = 64, 192 rows: T diag(beta) (rows 0-63),
constexpr int OFF_AQB = OFF_TB + 16384;          //   zeros (64-127), lower(Qp) (128-191)
constexpr int OFF_KD = OFF_TB + 24576;           // 2 x K e^{Gamma_last - Gamma} (by chunk parity)
constexpr int OFF_E = OFF_KD + 2 * 16384;        // E bf16 (MN-major, MN = v, K = j)
constexpr int OFF_S = OFF_E + 8192;              // S^T bf16 (MN-major, MN = v, K = c)
constexpr int OFF_SMALL = OFF_S + 16384;
constexpr int OFF_BETA = OFF_SMALL;              // fp32 [64]
constexpr int OFF_DECAY = OFF_BETA + 256;        // fp32 [2][128] e^{Gamma_last} (by chunk parity)
constexpr int OFF_BAR = OFF_DECAY + 1024;        // mbarriers + tmem base + flags
constexpr int OFF_DQ = OFF_BAR + 64;             // fp32 [64] d_k^{-1/2} q_i . k_i (exact)
constexpr int SMEM_USED = OFF_DQ + 256;
constexpr int SMEM_BYTES = SMEM_USED + 1024;     // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory over the sm_100 per-block limit");
static_assert(OFF_NS + 10 * 16 * LDX * 4 <= OFF_A + 65536, "phase-3 scratch overflows region A");
static_assert(OFF_RED + 16 <= OFF_A + 65536, "scan scratch overflows region A");
constexpr uint32_t TMEM_COLS = 512;

// TMEM columns.
constexpr uint32_t TM_GRAM = 0;     // all lanes  : Gram groups (cols 0-63 or 0-127)
constexpr uint32_t TM_UE = 128;     // all lanes  : rows 0-63 -K e^G S^T, rows 64-127 O
constexpr uint32_t TM_DS = 192;     // all lanes  : dS^T [c][v]
constexpr uint32_t TM_E = 256;      // all lanes  : rows 0-63 E = T diag(beta) (V - K e^G S^T)

struct TcParams {
    CUtensorMap map_k, map_q, map_v, map_g;
    ChunkArgs a;
};

template <int GATE>
__global__ void __launch_bounds__(NT, 1) kda_chunk_tc_kernel(const __grid_constant__ TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const ChunkArgs& a = p.a;
    const int H = a.H;
    const int vt = blockIdx.x % NVT;
    const int h = (blockIdx.x / NVT) % H;
    const int n = blockIdx.x / (NVT * H);
    const int hk = h / (H / a.Hk);     // query/key head (grouped value heads share it)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sp = warp & 3;           // TMEM sub-partition of this warp
    const int vhalf = warp >> 2;       // which 32 of the tile's 64 value columns
    const uint32_t lane_base = (uint32_t)(32 * sp) << 16;

    float* tot4 = reinterpret_cast<float*>(sm + OFF_TOT4);
    float* dq_s = reinterpret_cast<float*>(sm + OFF_DQ);
    float* gref_s = reinterpret_cast<float*>(sm + OFF_GREF);
    float* glast_s = reinterpret_cast<float*>(sm + OFF_GLAST);
    float* beta_s = reinterpret_cast<float*>(sm + OFF_BETA);
    float* decay_s = reinterpret_cast<float*>(sm + OFF_DECAY);
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint64_t* ut_bar = full_bar + 1;   // commits of the state-independent MMAs (Gram, W/U)
    uint64_t* st_bar = full_bar + 2;   // commits of the state MMAs (E/O1, O2/dS)
    uint64_t* v_bar = full_bar + 3;    // the V tile (waited only by the warps that read it)
    uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(full_bar + 4);
    int* abort_s = reinterpret_cast<int*>(full_bar + 5);
    const uint32_t sbase = smem_u32(sm);

    long long bos, eos;
    const bool seq_ok = seq_bounds(a.cu_seqlens, n, a.T, a.num_seqs, a.dev_status, bos, eos);
    if (!seq_ok) return;  // uniform across the CTA

    if (tid == 0) {
        mbar_init(full_bar, 1);
        mbar_init(ut_bar, 1);
        mbar_init(st_bar, 2);   // each state-MMA phase: two arrivals (kIssA, kIssB)
        mbar_init(v_bar, 1);
        *abort_s = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_base_s, TMEM_COLS);
        tmem_relinquish();
    }

    // ---- initial state: thread owns key channel c, value columns v0..v0+31
    const int c_own = 32 * sp + lane;
    const int v0 = 32 * vhalf;
    float S[32];
    {
        const size_t sbase_g = ((size_t)n * H + h) * DV * DK;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int v = vt * BV + v0 + j;
            S[j] = a.S0 ? a.S0[sbase_g + (size_t)v * DK + c_own] : 0.f;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
            st_shared_v4(sm + OFF_S, mnmaj_off(v0 + 8 * q, c_own, BV), pack8(S + 8 * q));
    }
    // the zero rows 64-127 of the T diag(beta) | 0 | lower(Qp) tile never change
    for (int e = tid; e < 512; e += NT)
        st_shared_v4(sm + OFF_TB + 8192, (uint32_t)(16 * e), make_uint4(0u, 0u, 0u, 0u));
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_base_s;

    // K, Q, g of a chunk complete on full_bar, V on v_bar.  Inside the chunk loop the
    // next chunk's tiles go out as soon as their buffers free: K and Q after the Gram
    // MMAs, g after the K|Q S^T MMAs, V after the E MMAs.
    auto issue_kq = [&](long long c1) {
        if (GATE == KDA_GATE_CHANNEL) mbar_expect_tx(full_bar, 32768u);   // g arrives later
        else mbar_arrive_expect_tx(full_bar, 32768u);
        tma_load_3d(sm + OFF_RK, &p.map_k, full_bar, 0, hk, (int)c1);
        tma_load_3d(sm + OFF_RQ, &p.map_q, full_bar, 0, hk, (int)c1);
    };
    auto issue_g = [&](long long c1) {
        mbar_arrive_expect_tx(full_bar, 32768u);
        tma_load_3d(sm + OFF_RG, &p.map_g, full_bar, 0, h, (int)c1);
    };
    auto issue_v = [&](long long c1) {
        mbar_arrive_expect_tx(v_bar, 8192u);
        tma_load_3d(sm + OFF_RV, &p.map_v, v_bar, vt * BV, h, (int)c1);
    };
    uint32_t full_phase = 0, ut_phase = 0, st_phase = 0, v_phase = 0;
    bool tma_pending = false, ut_pending = false, st_pending = false, v_pending = false;
    bool g_issued = true;   // the pending full_bar phase already has its arrival
    // Uniform bounded wait: every thread waits; any expiry aborts the CTA.
    // The phase flips only on success, so after an abort `phase` still names the
    // phase the cleanup has to wait for.
    auto wait_bar = [&](uint64_t* bar, uint32_t& phase) -> bool {
        const bool ok = mbar_wait(bar, phase, kWaitNs);
        if (!ok) atomicOr(abort_s, 1);
        __syncthreads();
        if (*abort_s != 0) return false;
        phase ^= 1u;
        return true;
    };

    if (tid == 0 && bos < eos) {
        issue_kq(bos);
        if (GATE == KDA_GATE_CHANNEL) issue_g(bos);
        issue_v(bos);
    }
    tma_pending = v_pending = bos < eos;

    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out);

    // Outputs and state update of a chunk whose O2 / dS MMAs have completed:
    // O rows go to HBM, S^T <- Diag(e^{Gamma_last}) S^T + dS^T (fp32 registers) and
    // its bf16 copy becomes the next chunk's MMA operand.
    auto finish_chunk = [&](long long cp, int Lp, const float* dec_buf) {
        const int i = 32 * (sp - 2) + lane;   // O rows live in lanes 64-127
        float v[32];
        if (sp >= 2) tmem_ld32(tm + lane_base + TM_UE + 32 * vhalf, v);
        if (sp >= 2 && i < Lp) {
            __nv_bfloat16* op = out + ((size_t)(cp + i) * H + h) * DV + vt * BV + 32 * vhalf;
#pragma unroll
            for (int q = 0; q < 4; ++q) reinterpret_cast<uint4*>(op)[q] = pack8(v + 8 * q);
        }
        float ds[32];
        tmem_ld32(tm + lane_base + TM_DS + 32 * vhalf, ds);
        const float dec = dec_buf[c_own];
#pragma unroll
        for (int jv = 0; jv < 32; ++jv) S[jv] = fmaf(S[jv], dec, ds[jv]);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            st_shared_v4(sm + OFF_S, mnmaj_off(v0 + 8 * q, c_own, BV), pack8(S + 8 * q));
    };

    bool aborted = false;
    long long c0_prev = 0;
    int L_prev = 0, par = 0;
    for (long long c0 = bos; c0 < eos; c0 += C, par ^= 1) {
        const int L = (int)min((long long)C, eos - c0);
        float* dec_cur = decay_s + par * DK;
        // ================= phase 1: log-space decay, reference factors, operands
        bool fast;   // one reference (chunk start) for the whole chunk, else 16-row sub-blocks
        const float beta_pf = (tid < L) ? a.beta[(size_t)(c0 + tid) * H + h] : 0.f;  // overlaps the wait
        if (!wait_bar(full_bar, full_phase)) { aborted = true; break; }
        tma_pending = false;
        {
            // thread tile: channels c8..c8+7 of rows 4 rg .. 4 rg + 3 (log2 units throughout)
            const int cq = tid & 15, rg = tid >> 4, c8 = 8 * cq;
            float g2[4][8], run[8];
            uint4 kraw[4], qraw[4];
#pragma unroll
            for (int e = 0; e < 8; ++e) run[e] = 0.f;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int i = 4 * rg + r;
                const bool valid = i < L;
                float gv[8];
                if (GATE == KDA_GATE_CHANNEL) {
                    const float4 a0 = *reinterpret_cast<const float4*>(sm + OFF_RG + (i * DK + c8) * 4);
                    const float4 a1 = *reinterpret_cast<const float4*>(sm + OFF_RG + (i * DK + c8 + 4) * 4);
                    gv[0] = a0.x; gv[1] = a0.y; gv[2] = a0.z; gv[3] = a0.w;
                    gv[4] = a1.x; gv[5] = a1.y; gv[6] = a1.z; gv[7] = a1.w;
                } else if (GATE == KDA_GATE_SCALAR) {
                    const float gs = valid ? a.g[(size_t)(c0 + i) * H + h] : 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) gv[e] = gs;
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) gv[e] = 0.f;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    run[e] += valid ? gv[e] * kLog2e : 0.f;
                    g2[r][e] = run[e];
                }
                const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
                kraw[r] = valid ? *reinterpret_cast<const uint4*>(sm + OFF_RK + (i * DK + c8) * 2) : z4;
                qraw[r] = valid ? *reinterpret_cast<const uint4*>(sm + OFF_RQ + (i * DK + c8) * 2) : z4;
            }
            *reinterpret_cast<float4*>(tot4 + rg * DK + c8) = make_float4(run[0], run[1], run[2], run[3]);
            *reinterpret_cast<float4*>(tot4 + rg * DK + c8 + 4) = make_float4(run[4], run[5], run[6], run[7]);
            if (tid < C) beta_s[tid] = beta_pf;
            // The diagonal of lower(Qp) is the undecayed q~_i . k_i.  Through the decayed
            // bf16 operands the cancellation in the channel sum would amplify their
            // rounding, so the operand loops below also form it from the raw inputs in fp32.
            float dqp[4];
            __syncthreads();   // raw K/Q/G are consumed; their space now takes operands
            // exclusive prefix over the 16 row groups, one thread per channel; the
            // reference row of sub-block b is row 16 b + 7 (prefix before group 4 b + 2)
            if (tid < DK) {
                float tv[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) tv[q] = tot4[q * DK + tid];
                float acc = 0.f;
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    if ((q & 3) == 2) gref_s[(q >> 2) * DK + tid] = acc;
                    const float t = tv[q];
                    tv[q] = acc;
                    acc += t;
                }
#pragma unroll
                for (int q = 0; q < 16; ++q) tot4[q * DK + tid] = tv[q];
                glast_s[tid] = acc;
                dec_cur[tid] = ex2(acc);
                float m = -acc;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                if (lane == 0) reinterpret_cast<float*>(sm + OFF_RED)[warp] = m;
            }
            __syncthreads();
            const float* red = reinterpret_cast<const float*>(sm + OFF_RED);
            fast = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])) <= kFastLimit2;
            const uint32_t basemn_f = (uint32_t)((rg >> 1) * 2048 + (cq >> 3) * 1024 + (rg & 1) * 512);
            if (fast) {
                // one reference: e^{Gamma_i} <= 1 on the i-side, e^{-Gamma_j} <= 2^112 on the j-side
                float pre[8], dec[8];
                {
                    const float4* pp = reinterpret_cast<const float4*>(tot4 + rg * DK + c8);
                    const float4* dp = reinterpret_cast<const float4*>(dec_cur + c8);
                    const float4 p0 = pp[0], p1 = pp[1], d0 = dp[0], d1 = dp[1];
                    pre[0] = p0.x; pre[1] = p0.y; pre[2] = p0.z; pre[3] = p0.w;
                    pre[4] = p1.x; pre[5] = p1.y; pre[6] = p1.z; pre[7] = p1.w;
                    dec[0] = d0.x; dec[1] = d0.y; dec[2] = d0.z; dec[3] = d0.w;
                    dec[4] = d1.x; dec[5] = d1.y; dec[6] = d1.z; dec[7] = d1.w;
                }
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const uint32_t omn = basemn_f + (((uint32_t)(cq & 7) ^ (uint32_t)(4 * (rg & 1) + r)) << 4) +
                                         (uint32_t)(r * 128);
                    float kf[8], qf[8], t1[8], t2[8], t3[8], t4[8];
                    unpack8(kraw[r], kf);
                    unpack8(qraw[r], qf);
                    dqp[r] = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        dqp[r] = fmaf(kf[e], qf[e], dqp[r]);
                        const float gm = pre[e] + g2[r][e];   // Gamma_i (log2), <= 0
                        const float eg = ex2(gm), ey = ex2(-gm);
                        t1[e] = kf[e] * eg;                    // K e^{Gamma}
                        t2[e] = -(qf[e] * a.scale) * eg;       // -Q~ e^{Gamma} (see phase 6)
                        t3[e] = kf[e] * ey;                    // K e^{-Gamma}
                        t4[e] = kf[e] * (dec[e] * ey);         // K e^{Gamma_last - Gamma}
                    }
                    st_shared_v4(sm + OFF_KQG, omn, pack8(t1));
                    st_shared_v4(sm + OFF_KQG, omn + 16384, pack8(t2));
                    st_shared_v4(sm + OFF_KYG, omn, pack8(t3));
                    st_shared_v4(sm + OFF_KD + par * 16384, omn, pack8(t4));
                }
            } else {
                const int b = rg >> 2;
                float pre[8], gr[8], Er[8], Lr[8], z[4][8];
                {
                    const float4* pp = reinterpret_cast<const float4*>(tot4 + rg * DK + c8);
                    const float4* gp = reinterpret_cast<const float4*>(gref_s + b * DK + c8);
                    const float4* lp = reinterpret_cast<const float4*>(glast_s + c8);
                    const float4 p0 = pp[0], p1 = pp[1], r0 = gp[0], r1 = gp[1], l0 = lp[0], l1 = lp[1];
                    const float pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
                    const float rv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
                    const float lv[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
    #pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        pre[e] = pv[e];
                        gr[e] = rv[e];
                        Er[e] = ex2(rv[e]);            // e^{Gamma_r}
                        Lr[e] = ex2(lv[e] - rv[e]);    // e^{Gamma_last - Gamma_r}
                    }
    #pragma unroll
                    for (int I = 1; I < 4; ++I) {
                        if (I > b) {
                            const float4* ip = reinterpret_cast<const float4*>(gref_s + I * DK + c8);
                            const float4 i0 = ip[0], i1 = ip[1];
                            const float iv[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
    #pragma unroll
                            for (int e = 0; e < 8; ++e) z[I][e] = ex2(iv[e] - rv[e]);   // e^{Gamma_rI - Gamma_r} <= 1
                        }
                    }
                }
                __syncthreads();   // the scan scratch shares region A with the j-side operands
                // swizzled byte offsets of this thread's 16-byte chunks (row i = 4 rg + r)
                const uint32_t sw0 = (uint32_t)(cq & 7);
                    // the same rows inside a 128-row tile (Gram A operands): K-atom stride 16 KB
                const uint32_t baseY = (uint32_t)((cq >> 3) * 16384 + (rg >> 1) * 1024 + (rg & 1) * 512);
                const uint32_t base128 = (uint32_t)((cq >> 3) * 16384 + ((rg >> 1) + 2 * b) * 1024 + (rg & 1) * 512);
                const uint32_t basemn = (uint32_t)((rg >> 1) * 2048 + (cq >> 3) * 1024 + (rg & 1) * 512);
    #pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const uint32_t swz = ((sw0 ^ (uint32_t)(4 * (rg & 1) + r)) << 4) + (uint32_t)(r * 128);
                    const uint32_t o128 = base128 + swz, omn = basemn + swz;
                    const uint32_t oy = baseY + swz;   // + (I >> 1) * 32768 + (I & 1) * 8192 for version I
                    float kf[8], qf[8], x[8], y[8], t[8];
                    unpack8(kraw[r], kf);
                    unpack8(qraw[r], qf);
                    dqp[r] = 0.f;
    #pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        dqp[r] = fmaf(kf[e], qf[e], dqp[r]);
                        const float dl = (pre[e] + g2[r][e]) - gr[e];   // Gamma_i - Gamma_r (log2)
                        x[e] = ex2(dl);
                        y[e] = ex2(-dl);
                        qf[e] *= a.scale;
                    }
                    // Gram i-side: K rows at 32 b + (i - 16 b), Q rows 16 further
    #pragma unroll
                    for (int e = 0; e < 8; ++e) t[e] = kf[e] * x[e];
                    st_shared_v4(sm + OFF_OX, o128, pack8(t));
    #pragma unroll
                    for (int e = 0; e < 8; ++e) t[e] = qf[e] * x[e];
                    st_shared_v4(sm + OFF_OX, o128 + 2048, pack8(t));
                    // Gram j-side for this sub-block and the later ones
                    float ky[8];
    #pragma unroll
                    for (int e = 0; e < 8; ++e) ky[e] = kf[e] * y[e];
                    st_shared_v4(sm + OFF_OY + (b >> 1) * 32768 + (b & 1) * 8192, oy, pack8(ky));
    #pragma unroll
                    for (int I = 1; I < 4; ++I) {
                        if (I > b) {
    #pragma unroll
                            for (int e = 0; e < 8; ++e) t[e] = ky[e] * z[I][e];
                            st_shared_v4(sm + OFF_OY + (I >> 1) * 32768 + (I & 1) * 8192, oy, pack8(t));
                        }
                    }
                    // K e^Gamma (MN-major), Q~ e^Gamma (K-major), K e^{Gamma_last - Gamma} (MN-major)
                    float t2[8];
    #pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float eg = Er[e] * x[e];
                        t[e] = kf[e] * eg;
                        t2[e] = -qf[e] * eg;
                    }
                    st_shared_v4(sm + OFF_KQG, omn, pack8(t));
                    st_shared_v4(sm + OFF_KQG, omn + 16384, pack8(t2));
    #pragma unroll
                    for (int e = 0; e < 8; ++e) t[e] = kf[e] * (Lr[e] * y[e]);
                    st_shared_v4(sm + OFF_KD + par * 16384, omn, pack8(t));
                }
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {   // 16 threads share a row
                float acc = dqp[r];
#pragma unroll
                for (int o = 1; o < 16; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                if (cq == 0) dq_s[4 * rg + r] = acc * a.scale;
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ================= phase 2: Gram MMAs.  Group g (M = 128, N = 64): A rows 0-63 are
        // the j-side operand of sub-block 2g, rows 64-127 that of sub-block 2g+1; B rows
        // are the i-side rows of sub-blocks 2g and 2g+1 (K then Q~ for each).
        // One-reference path: a single group, D[n][j] = [K e^G ; Q~ e^G]_n . (K e^-G)_j.
        if (tid == kGramTid) {
            if (fast) {
#pragma unroll
                for (int s8 = 0; s8 < 8; ++s8)
                    mma_bf16(tm + TM_GRAM, rowview_desc(sbase + OFF_KQG, s8),
                             rowview_desc(sbase + OFF_KYG, s8), idesc_bf16(128, 64, false, false),
                             s8 > 0);
            } else {
                const uint32_t ox = sbase + OFF_OX, oy = sbase + OFF_OY;
#pragma unroll
                for (int s8 = 0; s8 < 8; ++s8)
#pragma unroll
                    for (int g = 0; g < 2; ++g)
                        mma_bf16(tm + TM_GRAM + 64 * g, kmaj_desc(oy + g * 32768, 128, s8),
                                 kmaj_desc(ox + g * 8192, 128, s8), idesc_bf16(128, 64, false, false),
                                 s8 > 0);
            }
            mma_commit(ut_bar);
        }
        ut_pending = true;
        // while the Gram MMAs run: finish the previous chunk (its O2 / dS MMAs)
        if (st_pending) {
            if (!wait_bar(st_bar, st_phase)) { aborted = true; break; }
            st_pending = false;
            tc_fence_after();
            finish_chunk(c0_prev, L_prev, decay_s + (par ^ 1) * DK);
            fence_async_smem();
            tc_fence_before();
        }
        if (!wait_bar(ut_bar, ut_phase)) { aborted = true; break; }
        ut_pending = false;
        tc_fence_after();
        // S is current: [-K e^G S^T ; Q~ e^G S^T] with A = [K e^G ; -Q~ e^G] negated (M = 128).
        // It needs no T, so it runs while the coupling matrix is read out and inverted.
        if (tid == kIssA) {
            const uint32_t s_op = sbase + OFF_S;
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_bf16(tm + TM_UE, rowview_desc(sbase + OFF_KQG, s), mnmaj_desc(s_op, BV, s),
                         idesc_bf16(128, BV, false, true, true), s > 0);
            mma_commit(st_bar);
        } else if (tid == kIssB) {
            mbar_arrive(st_bar);
        }
        st_pending = true;
        const bool more = c0 + C < eos;
        if (tid == 32 && more) issue_kq(c0 + C);   // K|e^-G operand rows are consumed
        tma_pending = more;
        g_issued = !(more && GATE == KDA_GATE_CHANNEL);
        // ================= phase 3: coupling matrix L, lower(Qp), T = (I + L)^{-1}
        float* Lm = reinterpret_cast<float*>(sm + OFF_L);
        float* TF = reinterpret_cast<float*>(sm + OFF_TF);
        if (fast) {
            // lane n = 32 sp + lane: rows i of P (n < 64) or of Qp (n >= 64); warps 4-7
            // read all 64 columns j (warp 0 may still be issuing MMAs)
            if (vhalf == 1) {
                const int n = 32 * sp + lane;
#pragma unroll
                for (int hj = 0; hj < 2; ++hj) {
                    const int j0 = 32 * hj;
                    float v[32];
                    tmem_ld32(tm + lane_base + TM_GRAM + j0, v);
                    if (n < 64) {
                        const int i = n;
                        const float bi = beta_s[i];
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            float4 o;
                            o.x = (j0 + 4 * q + 0 < i) ? bi * v[4 * q + 0] : 0.f;
                            o.y = (j0 + 4 * q + 1 < i) ? bi * v[4 * q + 1] : 0.f;
                            o.z = (j0 + 4 * q + 2 < i) ? bi * v[4 * q + 2] : 0.f;
                            o.w = (j0 + 4 * q + 3 < i) ? bi * v[4 * q + 3] : 0.f;
                            *reinterpret_cast<float4*>(Lm + i * LDT + j0 + 4 * q) = o;
                        }
                    } else {
                        const int i = n - 64;
                        const float dii = dq_s[i];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            float t8[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const int j = j0 + 8 * q + e;
                                t8[e] = (j < i) ? -v[8 * q + e] : ((j == i) ? dii : 0.f);
                            }
                            st_shared_v4(sm + OFF_AQB, kmaj_off(i, j0 + 8 * q, 64), pack8(t8));
                        }
                    }
                }
            }
        } else {
            // warp group g reads Gram group g; lanes of sub-partitions 0-1 hold rows j of
            // sub-block 2g's version, those of 2-3 rows j of sub-block 2g+1's version
            const int g = vhalf, hi = sp >> 1;
            const int I = 2 * g + hi, j = 32 * (sp & 1) + lane;
            float* Q32 = reinterpret_cast<float*>(sm + OFF_Q32);
            float bi[16];
            {
                const float4* bp = reinterpret_cast<const float4*>(beta_s + 16 * I);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const float4 t4 = bp[q4];
                    bi[4 * q4] = t4.x; bi[4 * q4 + 1] = t4.y; bi[4 * q4 + 2] = t4.z; bi[4 * q4 + 3] = t4.w;
                }
            }
            float v[32];
            tmem_ld32(tm + lane_base + TM_GRAM + 64 * g + 32 * hi, v);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int i = 16 * I + u;
                Lm[i * LDT + j] = (j < i) ? bi[u] * v[u] : 0.f;
                Q32[i * LDT + j] = (j < i) ? v[16 + u] : ((j == i) ? dq_s[i] : 0.f);
            }
        }
        tc_fence_before();
        __syncthreads();
        // diagonal 16x16 blocks of T by forward substitution (lane = column)
        if (warp < 4) {
            const int I = warp, cc = lane & 15;
            float t[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int k = 0; k < r; ++k)
                    a4[k & 3] = fmaf(Lm[(16 * I + r) * LDT + 16 * I + k], t[k], a4[k & 3]);
                const float acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
                t[r] = (r < cc) ? 0.f : ((r == cc) ? 1.f : -acc);
            }
            if (lane < 16) {
#pragma unroll
                for (int r = 0; r < 16; ++r) TF[(16 * I + r) * LDT + 16 * I + cc] = t[r];
            }
        } else {
            if (sp < 2) {
                // E' = V - K e^G S^T, rows j = lanes 0-63, written over the V tile (MN-major)
                if (!mbar_wait(st_bar, st_phase, kWaitNs)) atomicOr(abort_s, 1);
                if (!mbar_wait(v_bar, v_phase, kWaitNs)) atomicOr(abort_s, 1);
                tc_fence_after();
                // the K e^G | -Q~ e^G tile is consumed: g of the next chunk can land there
                if (GATE == KDA_GATE_CHANNEL && tid == 128 && more) issue_g(c0 + C);
                const int j = 32 * sp + lane;
#pragma unroll
                for (int hv = 0; hv < 2; ++hv) {
                    float v[32];
                    tmem_ld32(tm + lane_base + TM_UE + 32 * hv, v);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t off = mnmaj_off(32 * hv + 8 * q, j, BV);
                        float vv[8];
                        unpack8(*reinterpret_cast<const uint4*>(sm + OFF_RV + off), vv);
#pragma unroll
                        for (int e = 0; e < 8; ++e) vv[e] += v[8 * q + e];
                        st_shared_v4(sm + OFF_RV, off, pack8(vv));
                    }
                }
                fence_async_smem();
            }
        }
        if (warp >= 4 && !fast) {
            // sub-block path: lower(Qp) -> bf16 operand
            for (int e = tid - 128; e < C * 8; e += 128) {
                const int i = e >> 3, j0 = 8 * (e & 7);
                const float* Q32 = reinterpret_cast<const float*>(sm + OFF_Q32);
                const float4 a0 = *reinterpret_cast<const float4*>(Q32 + i * LDT + j0);
                const float4 a1 = *reinterpret_cast<const float4*>(Q32 + i * LDT + j0 + 4);
                const float t8[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                st_shared_v4(sm + OFF_AQB, kmaj_off(i, j0, 64), pack8(t8));
            }
        }
        __syncthreads();
        if (*abort_s != 0) { aborted = true; break; }
        st_phase ^= 1u;    // the [-K e^G S^T ; O1] MMAs and the V tile were waited for above
        st_pending = false;
        v_phase ^= 1u;
        v_pending = false;
        tc_fence_before();
        // Off-diagonal blocks by a block Neumann series.  With D = blockdiag(T_II) and
        // N = D L_off (strictly block-lower, N^4 = 0):
        //   T = (I + N)^{-1} D = (I - N + N^2 - N^3) D,  so  T_IJ = M_IJ T_JJ (I > J)
        // with M = -N + N^2 - N^3.  Four levels of independent 16x16 products.
        {
            float* NS = reinterpret_cast<float*>(sm + OFF_NS);
            auto nb = [&](int idx) { return NS + idx * 16 * LDX; };
            auto tf = [&](int I, int J) { return TF + 16 * I * LDT + 16 * J; };
            auto lb = [&](int I, int J) { return Lm + 16 * I * LDT + 16 * J; };
            // N blocks: 0:(1,0) 1:(2,0) 2:(3,0) 3:(2,1) 4:(3,1) 5:(3,2); 6: N^2_20, 7: N^2_31,
            // 8: N^2_30, 9: N^3_30
            if (warp < 6) {
                const int I = (warp < 3) ? warp + 1 : ((warp < 5) ? warp - 1 : 3);
                const int K = (warp < 3) ? 0 : ((warp < 5) ? 1 : 2);
                float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                blk_mma(acc, tf(I, I), LDT, lb(I, K), LDT, lane);
                blk_store(nb(warp), LDX, acc, lane, 1.f);
            }
            __syncthreads();
            if (warp < 6) {
                float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                if (warp < 3) {   // T_{J+1,J} = -N_{J+1,J} T_JJ
                    const int J = warp, nidx = (J == 0) ? 0 : ((J == 1) ? 3 : 5);
                    blk_mma(acc, nb(nidx), LDX, tf(J, J), LDT, lane);
                    blk_store(tf(J + 1, J), LDT, acc, lane, -1.f);
                } else if (warp == 3) {   // N^2_20 = N_21 N_10
                    blk_mma(acc, nb(3), LDX, nb(0), LDX, lane);
                    blk_store(nb(6), LDX, acc, lane, 1.f);
                } else if (warp == 4) {   // N^2_31 = N_32 N_21
                    blk_mma(acc, nb(5), LDX, nb(3), LDX, lane);
                    blk_store(nb(7), LDX, acc, lane, 1.f);
                } else {                  // N^2_30 = N_31 N_10 + N_32 N_20
                    blk_mma(acc, nb(4), LDX, nb(0), LDX, lane);
                    blk_mma(acc, nb(5), LDX, nb(1), LDX, lane);
                    blk_store(nb(8), LDX, acc, lane, 1.f);
                }
            }
            __syncthreads();
            if (warp < 3) {
                float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                if (warp == 0) {          // T_20 = (N^2_20 - N_20) T_00
                    blk_mma2(acc, nb(6), 1.f, nb(1), -1.f, nullptr, 0.f, LDX, tf(0, 0), LDT, lane);
                    blk_store(tf(2, 0), LDT, acc, lane, 1.f);
                } else if (warp == 1) {   // T_31 = (N^2_31 - N_31) T_11
                    blk_mma2(acc, nb(7), 1.f, nb(4), -1.f, nullptr, 0.f, LDX, tf(1, 1), LDT, lane);
                    blk_store(tf(3, 1), LDT, acc, lane, 1.f);
                } else {                  // N^3_30 = N_32 N^2_20
                    blk_mma(acc, nb(5), LDX, nb(6), LDX, lane);
                    blk_store(nb(9), LDX, acc, lane, 1.f);
                }
            }
            __syncthreads();
            if (warp == 0) {              // T_30 = (N^2_30 - N_30 - N^3_30) T_00
                float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                blk_mma2(acc, nb(8), 1.f, nb(2), -1.f, nb(9), -1.f, LDX, tf(0, 0), LDT, lane);
                blk_store(tf(3, 0), LDT, acc, lane, 1.f);
            }
            __syncthreads();
        }
        // T diag(beta) -> bf16 operand rows 0-63 (K-major, K = j), 8 columns per step
        for (int e = tid; e < C * 8; e += NT) {
            const int i = e >> 3, j0 = 8 * (e & 7);
            const float4 a0 = *reinterpret_cast<const float4*>(TF + i * LDT + j0);
            const float4 a1 = *reinterpret_cast<const float4*>(TF + i * LDT + j0 + 4);
            const float4 b0 = *reinterpret_cast<const float4*>(beta_s + j0);
            const float4 b1 = *reinterpret_cast<const float4*>(beta_s + j0 + 4);
            const float tv[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
            float t8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) t8[k] = (j0 + k <= i) ? tv[k] * bv[k] : 0.f;
            st_shared_v4(sm + OFF_TB, kmaj_off(i, j0, 64), pack8(t8));
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ================= phase 4: [E ; 0] = [T diag(beta) ; 0] E'  (M = 128, K = 64)
        if (tid == kIssB) {
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_bf16(tm + TM_E, kmaj_desc(sbase + OFF_TB, 128, s), mnmaj_desc(sbase + OFF_RV, 64, s),
                         idesc_bf16(128, 64, false, true), s > 0);
            mma_commit(ut_bar);
        }
        ut_pending = true;
        if (!wait_bar(ut_bar, ut_phase)) { aborted = true; break; }
        ut_pending = false;
        tc_fence_after();
        // E' (written over V) is consumed: the next chunk's V completes the TMA phase
        if (tid == kIssB && more) issue_v(c0 + C);
        v_pending = more;
        g_issued = true;
        // ================= phase 7: E -> bf16 (MN-major, MN = v, K = j); E rows are lanes 0-63
        if (sp < 2) {
            const int j = 32 * sp + lane;
            float v[32];
            tmem_ld32(tm + lane_base + TM_E + 32 * vhalf, v);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                st_shared_v4(sm + OFF_E, mnmaj_off(32 * vhalf + 8 * q, j, BV), pack8(v + 8 * q));
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ================= phase 8: O += lower(Qp) E ; dS^T = (K e^{G_last - G})^T E
        // (issued without waiting: the next chunk's prep runs while they execute)
        if (tid == kIssA) {
            const uint32_t e_op = sbase + OFF_E;
#pragma unroll
            for (int s = 0; s < 4; ++s)   // rows 64-127: O += lower(Qp) E; rows 0-63 add zero
                mma_bf16(tm + TM_UE, kmaj_desc(sbase + OFF_TB + 8192, 128, s), mnmaj_desc(e_op, BV, s),
                         idesc_bf16(128, BV, false, true), 1);
            mma_commit(st_bar);
        } else if (tid == kIssB) {
            const uint32_t e_op = sbase + OFF_E;
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_bf16(tm + TM_DS, mnmaj_desc(sbase + OFF_KD + par * 16384, 128, s),
                         mnmaj_desc(e_op, BV, s), idesc_bf16(128, BV, true, true), s > 0);
            mma_commit(st_bar);
        }
        st_pending = true;
        c0_prev = c0;
        L_prev = L;
    }
    if (!aborted && st_pending) {
        if (!wait_bar(st_bar, st_phase)) {
            aborted = true;
        } else {
            st_pending = false;
            tc_fence_after();
            finish_chunk(c0_prev, L_prev, decay_s + (par ^ 1) * DK);
        }
    }

    if (aborted) {
        if (a.dev_status && tid == 0) atomicOr(a.dev_status, KDA_DEV_TIMEOUT);
        // let copies / MMAs still in flight land before the memory goes away
        if (tma_pending) {
            if (tid == 0 && !g_issued) mbar_arrive(full_bar);   // let the landed bytes close it
            (void)mbar_wait(full_bar, full_phase, kWaitNs);
        }
        if (v_pending) (void)mbar_wait(v_bar, v_phase, kWaitNs);
        if (ut_pending) (void)mbar_wait(ut_bar, ut_phase, kWaitNs);
        if (st_pending) (void)mbar_wait(st_bar, st_phase, kWaitNs);
    } else if (a.S_T) {
        const size_t sbase_g = ((size_t)n * H + h) * DV * DK;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int v = vt * BV + v0 + j;
            a.S_T[sbase_g + (size_t)v * DK + c_own] = S[j];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side

template <int GATE>
cudaError_t launch_gate(const TcParams& p, int grid, cudaStream_t st) {
    auto kern = kda_chunk_tc_kernel<GATE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<grid, NT, SMEM_BYTES, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool chunk_tc_supported(int D, int V, int Cc) { return D == DK && V == DV && Cc == C; }

cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t st) {
    TcParams p;
    memset(&p, 0, sizeof(p));
    p.a = a;
    const long long tokens = (long long)a.B * a.T;
    if (tokens > 0) {  // with no tokens the kernel only copies S0 to S_T and never issues TMA
        bool ok = make_map(&p.map_k, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, a.Hk, tokens, DK,
                           C, CU_TENSOR_MAP_SWIZZLE_NONE) &&
                  make_map(&p.map_q, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, a.Hk, tokens, DK,
                           C, CU_TENSOR_MAP_SWIZZLE_NONE) &&
                  make_map(&p.map_v, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DV, a.H, tokens, BV,
                           C, CU_TENSOR_MAP_SWIZZLE_128B);
        if (ok && a.gate == KDA_GATE_CHANNEL)
            ok = make_map(&p.map_g, a.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, DK, a.H, tokens, DK, C,
                          CU_TENSOR_MAP_SWIZZLE_NONE);
        if (!ok) return cudaErrorInvalidValue;
    }
    const int grid = a.num_seqs * a.H * NVT;
    switch (a.gate) {
        case KDA_GATE_CHANNEL: return launch_gate<KDA_GATE_CHANNEL>(p, grid, st);
        case KDA_GATE_SCALAR: return launch_gate<KDA_GATE_SCALAR>(p, grid, st);
        default: return launch_gate<KDA_GATE_NONE>(p, grid, st);
    }
}

}  // namespace kda
