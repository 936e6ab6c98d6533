// kda_chunk_wy.cu -- the state-independent half of the two-kernel
// tensor-core prefill: one CTA per (chunk, head) computes the log-space
// cumulative decay, the decay-masked key/key and query/key products (tcgen05
// MMAs), the unit-lower-triangular inverse T = (I + L)^{-1} and the WY/UT
// pseudo-value products W and U^T, and writes them as a record (layout in
// kda_chunk_record.cuh).  Chunks are independent, so the whole grid runs in
// parallel; only the state scan that follows is sequential.
//
// Chunkwise form: GeekNews summary of "You could have come up with Kimi
// Delta Attention", section "Chunkwise KDA" (cumulative decay, coupling of
// the in-chunk errors); the triangular solve into pseudo-values is the one
// the curriculum page names ("WY/UT form").  For a chunk of C tokens:
//
//   Gamma_i = sum_{s<=i} g_s                                   (log2 units)
//   P[i,j]  = sum_c K_ic K_jc 2^{Gamma_ic - Gamma_jc}    L = strict_lower(diag(beta) P)
//   Qp[i,j] = sum_c Q~_ic K_jc 2^{Gamma_ic - Gamma_jc}   T = (I + L)^{-1}
//
// Two ways to split 2^{Gamma_i - Gamma_j} into an i-side and a j-side factor:
//  * one reference (chunk start): i-side 2^{Gamma_i} <= 1, j-side 2^{-Gamma_j},
//    used while max_c |Gamma_last,c| <= 112 so that the j-side stays finite;
//  * sub-block references (16-token sub-blocks, reference row r(I)): i-side
//    2^{Gamma_i - Gamma_r(I)}, j-side 2^{Gamma_r(I) - Gamma_j} (one version of
//    the j-side per sub-block I), bounded for any decay a token can carry.
// The fast kernel takes every chunk; a chunk that needs sub-block references
// is put on a list that the slow kernel (more shared memory, one CTA per SM)
// works through afterwards.
//
// Precision.  The decay factors span far more than fp16's exponent range, so
// the Gram operands are bf16; the query rows and the j-side are each carried
// as a two-term bf16 expansion (hi + lo, about 16 significant bits), and the
// products hi*hi + hi*lo + lo*hi are summed in the fp32 accumulator, so Qp
// keeps close to fp32 accuracy (the key rows, which only feed L, use one
// term).  T diag(beta) is split the same way for the W and U products, whose
// other operands (K e^{Gamma} in bf16, the raw bf16 values) are used as they
// are.  Everything the record carries is fp16.
#include <cudaTypedefs.h>

#include "kda_chunk_record.cuh"
#include "kda_internal.cuh"
#include "kda_tc_common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;
using namespace tc;

constexpr int C = rec::C, DK = rec::DK, NT = 256;
constexpr uint64_t kWaitNs = 1000000000ull;   // 1 s bound on every wait
constexpr float kFastLimit2 = 112.f;          // one reference while max |Gamma_last| <= 112 (log2)
// Two references while every 16-row sub-block's decay is <= 100 (log2): an i-side factor of
// a row of half 1 over row 15 that underflows then meets a j-side factor <= 2^100, so the
// product it drops is below 2^-26.
constexpr float kTwoLimit2 = 100.f;
constexpr int LDT = 68;                       // fp32 row stride of L and T (bank spread)
constexpr int LDX = 20;                       // fp32 row stride of 16x16 block scratch
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t TM_GRAM = 0;               // Gram: 128 columns (two accumulator regions)
constexpr uint32_t TM_UT = 0;                 // U^T hi and lo terms (M = 128, N = 128), after the Gram is read out
constexpr uint32_t TM_W = 128;                // W (M = 64: lanes 0-15 of each sub-partition)

// Shared-memory maps (bytes from a 1024-aligned base).
template <bool SLOW>
struct WyMap;
template <>
struct WyMap<false> {                          // one-reference chunks, two CTAs per SM
    static constexpr int RK = 0, RQ = 16384, RG = 32768, RV = 81920;   // raw K, Q, g, V (2 tiles)
    // after prep: rows 0-63 K e^G, 64-127 Q~ e^G (hi), 128-191 Q~ e^G (lo), each (row r,
    // channel c) at mnmaj_off(c, r, 128); rows 0-63 are also the B operand of W
    static constexpr int KQ3 = 0;
    static constexpr int KY = 49152;           //   rows 0-63 K e^{-G} (hi), rows 64-127 its lo term
    static constexpr int KG = KQ3;
    static constexpr int TOT4 = 98304;         // decay scan scratch (prep only)
    // GREF: the two-reference terms per channel, rows G_r0, G_r1, 2^{G_r0}, 2^{G_r1},
    // 2^{G_last - G_r0}, 2^{G_last - G_r1}
    static constexpr int GREF = TOT4 + 8192, GLAST = GREF + 3072, RED = GLAST + 512;
    static constexpr int L = 16384;            // after the Gram: fp32 L, T, Neumann blocks
    static constexpr int TF = L + 64 * LDT * 4;
    static constexpr int NS = TF + 64 * LDT * 4;
    static constexpr int AQST = 65536;         // fp16 lower(Qp) staging (over the lo j-side)
    // T diag(beta), hi then lo (bf16, K-major, 64 rows each: one 128-row tile), over the
    // lower(Qp) staging once its bulk store has read it
    static constexpr int TB = 65536, TBL = TB + 8192;
    static constexpr int WST = 16384, UST = 32768;  // after the W/U MMAs: record images of W, U^T
    static constexpr int OX = 0, OXL = 0, OY = 0, OYL = 0;   // sub-block path only
    static constexpr int DECS = RED + 64, BETA = DECS + 512, BAR = BETA + 256, DQS = BAR + 64;
    static constexpr int END = DQS + 256;
    static_assert(NS + 10 * 16 * LDX * 4 <= KY + 16384, "phase-3 scratch overflows into the lo j-side");
    static_assert(KY + 32768 <= RV && RV + 16384 <= TOT4, "operands overlap V");
    static_assert(TBL + 8192 <= RV, "T diag(beta) overlaps V");
};
template <>
struct WyMap<true> {                           // sub-block references, one CTA per SM
    static constexpr int RK = 0, RQ = 16384, RG = 32768, RV = 65536;
    static constexpr int OX = 0;               // after prep: Gram i-side rows (K-major, 128 rows)
    static constexpr int KG = 32768;           //   K e^G (MN-major, MN = channel)
    static constexpr int OXL = 49152;          //   Q~ i-side rows (lo), K-major, 64 rows
    static constexpr int A = 81920;            // 64 KB, reused: scan scratch, Gram j-side (hi)
    static constexpr int TOT4 = A, GREF = TOT4 + 8192, GLAST = GREF + 2048, RED = GLAST + 512;
    static constexpr int OY = A;               //   2 K-major tiles of 128 rows (versions 2g, 2g+1)
    static constexpr int OYL = A + 65536;      //   the same, lo terms
    static constexpr int L = A;                //   after the Gram: fp32 L, T, Neumann blocks,
    static constexpr int TF = L + 64 * LDT * 4;
    static constexpr int NS = TF + 64 * LDT * 4;
    static constexpr int AQST = NS + 10 * 16 * LDX * 4;   // fp16 lower(Qp) staging
    static constexpr int TB = OYL, TBL = TB + 8192;
    static constexpr int KQ3 = 0, KY = 0;      // one-reference path only
    static constexpr int WST = A, UST = A + 16384;   // after the W/U MMAs: record images of W, U^T
    static_assert(UST + 16384 <= AQST, "W/U staging overlaps the lower(Qp) staging");
    static constexpr int DECS = OYL + 65536, BETA = DECS + 512, BAR = BETA + 256, DQS = BAR + 64;
    static constexpr int END = DQS + 256;
    static_assert(AQST + 8192 <= OYL, "phase-3 scratch overflows region A");
};
template <bool SLOW>
constexpr int wy_smem_bytes() { return WyMap<SLOW>::END + 1024; }
static_assert(2 * (wy_smem_bytes<false>() + 1024) <= 233472, "fast kernel must fit twice per SM");
static_assert(wy_smem_bytes<true>() <= 232448, "shared memory over the sm_100 per-block limit");

struct WyParams {
    CUtensorMap map_k, map_q, map_v, map_g;
    const float* g;
    const float* beta;
    const int32_t* cu_seqlens;
    const int32_t* coff;      // packed batches: first slot of each sequence, [num_seqs + 1]
    int32_t* slow;            // [0] count, [1 + x] = slot * H + head
    int32_t* dev_status;
    uint8_t* rec;
    int T, H, num_seqs, nc;   // nc: slots per sequence of a dense batch
    int ahead;                // fast kernel: L2 prefetch distance in CTAs (one per SM)
    int group;                // value heads per query/key head (q/k head of h: h / group)
    float scale;
};

// Slot -> (sequence, first row, length).  False for slots past the last chunk.
__device__ __forceinline__ bool decode_slot(const WyParams& p, int slot, long long& c0, int& L) {
    long long bos, eos, first;
    if (p.cu_seqlens == nullptr) {
        const int n = slot / p.nc;
        bos = (long long)n * p.T;
        eos = bos + p.T;
        first = (long long)n * p.nc;
    } else {
        if (slot >= p.coff[p.num_seqs]) return false;
        int lo = 0, hi = p.num_seqs - 1;   // largest n with coff[n] <= slot
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.coff[mid] <= slot) lo = mid; else hi = mid - 1;
        }
        bos = p.cu_seqlens[lo];
        eos = p.cu_seqlens[lo + 1];
        first = p.coff[lo];
    }
    c0 = bos + (slot - first) * C;
    L = (int)min((long long)C, eos - c0);
    return L > 0;
}

// Off-diagonal 16x16 blocks of T = (I + L)^{-1} from its diagonal blocks T_II, one
// block column per warp (forward substitution by blocks):
//   T_IJ = -T_II sum_{K=J}^{I-1} L_IK T_KJ        (I > J),
// each product a 16x16 warp-level tf32 MMA; P is warp-private scratch.  Column 0
// is the longest chain (T10 -> T20 -> T30): warp 3, on the fourth sub-partition,
// takes its terms that wait for nothing or only for T10 (L20 T00, L30 T00 + L31 T10)
// and hands them over through named barriers, in the summation order of the
// plain column loop.
__device__ __forceinline__ void named_sync(int id) {
    asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory");
}
__device__ __forceinline__ void named_arrive(int id) {
    asm volatile("bar.arrive %0, 64;" ::"r"(id) : "memory");
}
// The C-fragment pair that blk_store writes, read back.
__device__ __forceinline__ void blk_load(float (&acc)[2][4], const float* Cm, int ld, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        acc[nt][0] = Cm[g * ld + 8 * nt + 2 * t];
        acc[nt][1] = Cm[g * ld + 8 * nt + 2 * t + 1];
        acc[nt][2] = Cm[(g + 8) * ld + 8 * nt + 2 * t];
        acc[nt][3] = Cm[(g + 8) * ld + 8 * nt + 2 * t + 1];
    }
}
__device__ __forceinline__ void offdiag_columns(float* TF, const float* Lm, float* NS, int warp,
                                                int lane) {
    auto tf = [&](int I, int J) { return TF + 16 * I * LDT + 16 * J; };
    auto lb = [&](int I, int J) { return Lm + 16 * I * LDT + 16 * J; };
    auto finish = [&](float (&acc)[2][4], float* P, int I, int J) {   // T_IJ = -T_II acc
        blk_store(P, LDX, acc, lane, 1.f);
        __syncwarp();
        float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        blk_mma(acc2, tf(I, I), LDT, P, LDX, lane);
        blk_store(tf(I, J), LDT, acc2, lane, -1.f);
        __syncwarp();
    };
    float* XA = NS + 3 * 16 * LDX;   // L20 T00
    float* XB = NS + 4 * 16 * LDX;   // L30 T00 + L31 T10
    if (warp == 0) {
        float* P = NS;
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        blk_mma(acc, lb(1, 0), LDT, tf(0, 0), LDT, lane);
        finish(acc, P, 1, 0);
        named_arrive(1);   // T10 ready
        named_sync(2);     // L20 T00 ready
        blk_load(acc, XA, LDX, lane);
        blk_mma(acc, lb(2, 1), LDT, tf(1, 0), LDT, lane);
        finish(acc, P, 2, 0);
        named_sync(3);     // L30 T00 + L31 T10 ready
        blk_load(acc, XB, LDX, lane);
        blk_mma(acc, lb(3, 2), LDT, tf(2, 0), LDT, lane);
        finish(acc, P, 3, 0);
    } else if (warp == 3) {
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        blk_mma(acc, lb(2, 0), LDT, tf(0, 0), LDT, lane);
        blk_store(XA, LDX, acc, lane, 1.f);
        float accb[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        blk_mma(accb, lb(3, 0), LDT, tf(0, 0), LDT, lane);
        named_arrive(2);
        named_sync(1);
        blk_mma(accb, lb(3, 1), LDT, tf(1, 0), LDT, lane);
        blk_store(XB, LDX, accb, lane, 1.f);
        named_arrive(3);
    } else if (warp < 3) {
        const int J = warp;
        float* P = NS + warp * 16 * LDX;
        for (int I = J + 1; I < 4; ++I) {
            float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            for (int K = J; K < I; ++K) blk_mma(acc, lb(I, K), LDT, tf(K, J), LDT, lane);
            finish(acc, P, I, J);
        }
    }
    __syncthreads();
}

// One (chunk, head).  Returns 0 when the record is written, 1 when the chunk
// needs sub-block references (fast kernel only; nothing written), 2 when a
// bounded wait expired (everything in flight has been waited for again).
template <int GATE, bool SLOW>
__device__ __forceinline__ int wy_job(const WyParams& p, uint8_t* sm, uint32_t tm, int slot, int h,
                                      uint32_t& full_phase, uint32_t& mma_phase, uint32_t& v_phase) {
    using M = WyMap<SLOW>;
    const int H = p.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sp = warp & 3, half = warp >> 2;
    const uint32_t lane_base = (uint32_t)(32 * sp) << 16;
    const uint32_t sbase = smem_u32(sm);
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(sm + M::BAR);
    uint64_t* mma_bar = full_bar + 1;
    uint64_t* v_bar = full_bar + 4;   // the V tiles, needed only by the U MMAs
    volatile int* flag_s = reinterpret_cast<volatile int*>(full_bar + 3);
    float* tot4 = reinterpret_cast<float*>(sm + M::TOT4);
    float* gref_s = reinterpret_cast<float*>(sm + M::GREF);
    float* glast_s = reinterpret_cast<float*>(sm + M::GLAST);
    float* dec_s = reinterpret_cast<float*>(sm + M::DECS);
    float* beta_s = reinterpret_cast<float*>(sm + M::BETA);
    float* dq_s = reinterpret_cast<float*>(sm + M::DQS);   // d_k^{-1/2} q_i . k_i, exact in fp32

    long long c0;
    int L;
    if (!decode_slot(p, slot, c0, L)) return 0;
    uint8_t* rec_p = p.rec + ((size_t)slot * H + h) * rec::BYTES;

    // Uniform bounded wait: on expiry every thread leaves with `false` after
    // waiting once more for the same phase (copies / MMAs still in flight).
    bool v_pending = false;   // the V copy is in flight (every exit waits for it)
    auto wait_v = [&]() {
        if (v_pending) {
            if (!mbar_wait(v_bar, v_phase, kWaitNs)) *flag_s = 1;
            v_phase ^= 1u;
            v_pending = false;
        }
    };
    auto wait_all = [&](uint64_t* bar, uint32_t& phase) -> bool {
        if (!mbar_wait(bar, phase, kWaitNs)) *flag_s = 1;
        __syncthreads();
        if (*flag_s != 0) {
            (void)mbar_wait(bar, phase, kWaitNs);
            wait_v();
            if (p.dev_status && tid == 0) atomicOr(p.dev_status, KDA_DEV_TIMEOUT);
            return false;
        }
        phase ^= 1u;
        return true;
    };

    if (tid == 0) {
        // K, Q (16 KB each), per-channel g (32 KB); V (two 8 KB tiles) on its own barrier
        const uint32_t bytes = 16384u * 2u + (GATE == KDA_GATE_CHANNEL ? 32768u : 0u);
        mbar_arrive_expect_tx(full_bar, bytes);
        tma_load_3d(sm + M::RK, &p.map_k, full_bar, 0, h / p.group, (int)c0);
        tma_load_3d(sm + M::RQ, &p.map_q, full_bar, 0, h / p.group, (int)c0);
        if (GATE == KDA_GATE_CHANNEL) tma_load_3d(sm + M::RG, &p.map_g, full_bar, 0, h, (int)c0);
        mbar_arrive_expect_tx(v_bar, 16384u);
        tma_load_3d(sm + M::RV, &p.map_v, v_bar, 0, h, (int)c0);
        tma_load_3d(sm + M::RV + 8192, &p.map_v, v_bar, 64, h, (int)c0);
        if (!SLOW) {
            // the job p.ahead blocks later (blocks start in linear order): its tiles go
            // to L2 now, so that its own loads hit there
            const long long lin = blockIdx.x + (long long)blockIdx.y * gridDim.x + p.ahead;
            long long c2;
            int L2;
            if (lin < (long long)gridDim.x * gridDim.y &&
                decode_slot(p, (int)(lin % gridDim.x), c2, L2)) {
                const int h2 = (int)(lin / gridDim.x);
                tma_prefetch_l2_3d(&p.map_k, 0, h2 / p.group, (int)c2);
                tma_prefetch_l2_3d(&p.map_q, 0, h2 / p.group, (int)c2);
                tma_prefetch_l2_3d(&p.map_v, 0, h2, (int)c2);
                tma_prefetch_l2_3d(&p.map_v, 64, h2, (int)c2);
                if (GATE == KDA_GATE_CHANNEL) tma_prefetch_l2_3d(&p.map_g, 0, h2, (int)c2);
            }
        }
    }
    v_pending = true;
    const float beta_pf = (tid < L) ? p.beta[(size_t)(c0 + tid) * H + h] : 0.f;
    // One gate value per token (or none) in the one-reference kernel: the decay is a
    // per-row factor, so the cumulative sum runs over 64 values instead of 64 x 128.
    constexpr bool ROWGATE = !SLOW && GATE != KDA_GATE_CHANNEL;
    const float gsc_pf = (ROWGATE && GATE == KDA_GATE_SCALAR && tid < L)
                             ? p.g[(size_t)(c0 + tid) * H + h] * kLog2e : 0.f;
    if (!wait_all(full_bar, full_phase)) return 2;

    // ================= log-space decay: thread tile = channels c8..c8+7 of rows 4 rg .. 4 rg + 3
    bool fast;
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
        if (ROWGATE) {
#pragma unroll
            for (int e = 0; e < 8; ++e) gv[e] = 0.f;   // handled per row below
        } else if (GATE == KDA_GATE_CHANNEL) {
            const float4 a0 = *reinterpret_cast<const float4*>(sm + M::RG + (i * DK + c8) * 4);
            const float4 a1 = *reinterpret_cast<const float4*>(sm + M::RG + (i * DK + c8 + 4) * 4);
            gv[0] = a0.x; gv[1] = a0.y; gv[2] = a0.z; gv[3] = a0.w;
            gv[4] = a1.x; gv[5] = a1.y; gv[6] = a1.z; gv[7] = a1.w;
        } else if (GATE == KDA_GATE_SCALAR) {
            const float gs = valid ? p.g[(size_t)(c0 + i) * H + h] : 0.f;
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
        kraw[r] = valid ? *reinterpret_cast<const uint4*>(sm + M::RK + (i * DK + c8) * 2) : z4;
        qraw[r] = valid ? *reinterpret_cast<const uint4*>(sm + M::RQ + (i * DK + c8) * 2) : z4;
    }
    if (!ROWGATE) {
        *reinterpret_cast<float4*>(tot4 + rg * DK + c8) = make_float4(run[0], run[1], run[2], run[3]);
        *reinterpret_cast<float4*>(tot4 + rg * DK + c8 + 4) = make_float4(run[4], run[5], run[6], run[7]);
    }
    // The diagonal of lower(Qp) is the undecayed q~_i . k_i.  Through the decayed bf16
    // operands it would carry their rounding amplified by the cancellation in the
    // channel sum, so the operand loops below also form it from the raw inputs in fp32.
    float dqp[4];
    auto store_dq = [&]() {   // all threads; 16 threads share a row
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            float acc = dqp[r];
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (cq == 0) dq_s[4 * rg + r] = acc * p.scale;
        }
    };
    if (tid < C) beta_s[tid] = beta_pf;
    float* rowf = tot4;        // per-row gate factors 2^{Gamma_i}, 2^{-Gamma_i} (ROWGATE)
    float* rowi = tot4 + C;
    float* red = reinterpret_cast<float*>(sm + M::RED);
    if (ROWGATE && GATE == KDA_GATE_SCALAR) {
        // inclusive scan of the per-token log2 decay over the 64 rows (two warps)
        float x = gsc_pf;
        if (tid < C) {
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (lane == 31) red[warp] = x;
        }
        __syncthreads();
        if (tid < C) {
            if (warp == 1) x += red[0];
            rowf[tid] = ex2(x);
            rowi[tid] = ex2(-x);   // only used when the chunk takes one reference
            if (tid == C - 1) red[2] = x;
        }
    }
    __syncthreads();   // raw K / Q / g are consumed; their space now takes operands
    if (ROWGATE) {
        const float glast = (GATE == KDA_GATE_SCALAR) ? red[2] : 0.f;
        fast = -glast <= kFastLimit2;
        if (tid < DK) {
            const float d = (GATE == KDA_GATE_SCALAR) ? ex2(glast) : 1.f;
            dec_s[tid] = d;
            reinterpret_cast<float*>(rec_p + rec::DEC)[tid] = d;
        }
    }
    // exclusive prefix over the 16 row groups, one thread per channel.  Sub-block
    // kernel: the reference row of sub-block b is row 16 b + 7 (prefix before group
    // 4 b + 2).  One-reference kernel: the two-reference form's rows 15 and 47 (prefix
    // before groups 4 and 12) and 2^{Gamma_15}.
    if (!ROWGATE && tid < DK) {
        float tv[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) tv[q] = tot4[q * DK + tid];
        float acc = 0.f;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            if (SLOW && (q & 3) == 2) gref_s[(q >> 2) * DK + tid] = acc;
            const float t = tv[q];
            tv[q] = acc;
            acc += t;
        }
#pragma unroll
        for (int q = 0; q < 16; ++q) tot4[q * DK + tid] = tv[q];
        glast_s[tid] = acc;
        if (!SLOW) {
            gref_s[tid] = tv[4];
            gref_s[DK + tid] = tv[12];
            gref_s[2 * DK + tid] = ex2(tv[4]);
            gref_s[3 * DK + tid] = ex2(tv[12]);
            gref_s[4 * DK + tid] = ex2(acc - tv[4]);
            gref_s[5 * DK + tid] = ex2(acc - tv[12]);
        }
        const float d = ex2(acc);
        dec_s[tid] = d;
        reinterpret_cast<float*>(rec_p + rec::DEC)[tid] = d;
        // the chunk's decay, and the largest decay of one 16-row sub-block
        float m = -acc, mb = fmaxf(fmaxf(-tv[4], tv[4] - tv[8]), fmaxf(tv[8] - tv[12], tv[12] - acc));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
        }
        if (lane == 0) {
            reinterpret_cast<float*>(sm + M::RED)[warp] = m;
            reinterpret_cast<float*>(sm + M::RED)[4 + warp] = mb;
        }
    }
    __syncthreads();
    // Two references (one-reference kernel, per-channel gate): rows 15 and 47, each the
    // reference of its 32-row half, for chunks whose decay is too large for one reference
    // but within bounds over every 16-row sub-block.
    // (re-read from shared memory where it is needed again: no register carries it)
    auto two_ref = [&]() -> bool {
        if (ROWGATE || SLOW) return false;
        const volatile float* rv = red;
        return fmaxf(fmaxf(rv[0], rv[1]), fmaxf(rv[2], rv[3])) > kFastLimit2 &&
               fmaxf(fmaxf(rv[4], rv[5]), fmaxf(rv[6], rv[7])) <= kTwoLimit2;
    };
    const bool two = two_ref();
    if (!ROWGATE) fast = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])) <= kFastLimit2;
    if (!SLOW && !fast && !two) {
        if (tid == 0) {
            const int pos = atomicAdd(p.slow, 1);
            p.slow[1 + pos] = slot * H + h;
        }
        wait_v();          // no copy may land after the CTA is gone
        __syncthreads();   // the scratch of this job is read no more
        return 1;
    }
    uint8_t* g_wq = rec_p + rec::WQ;
    uint8_t* g_kd = rec_p + rec::KD;
    // the 16-byte chunks of this thread: (row 4 rg + r, channels c8..c8+7) in the
    // mnmaj_off(c, row, 128) layout shared by K e^G, Q~ e^G, K e^{-G}, Qg and Kd
    const uint32_t basemn = (uint32_t)((rg >> 1) * 2048 + (cq >> 3) * 1024 + (rg & 1) * 512);
    if (!SLOW && !two) {
        // ================= one reference: 2^{Gamma_i} <= 1 on the i-side, 2^{-Gamma_j} <= 2^112 on
        // the j-side; one decay per row when the gate is scalar or absent
        float pre[8], dec[8];
        if (!ROWGATE) {
            const float4* pp = reinterpret_cast<const float4*>(tot4 + rg * DK + c8);
            const float4* dp = reinterpret_cast<const float4*>(dec_s + c8);
            const float4 p0 = pp[0], p1 = pp[1], d0 = dp[0], d1 = dp[1];
            pre[0] = p0.x; pre[1] = p0.y; pre[2] = p0.z; pre[3] = p0.w;
            pre[4] = p1.x; pre[5] = p1.y; pre[6] = p1.z; pre[7] = p1.w;
            dec[0] = d0.x; dec[1] = d0.y; dec[2] = d0.z; dec[3] = d0.w;
            dec[4] = d1.x; dec[5] = d1.y; dec[6] = d1.z; dec[7] = d1.w;
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int i = 4 * rg + r;
            const uint32_t omn =
                basemn + (((uint32_t)(cq & 7) ^ (uint32_t)(4 * (rg & 1) + r)) << 4) + (uint32_t)(r * 128);
            float kf[8], qf[8], kx[8], qx[8], ky[8], kd[8];
            unpack8(kraw[r], kf);
            unpack8(qraw[r], qf);
            dqp[r] = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                dqp[r] = fmaf(kf[e], qf[e], dqp[r]);
                float eg, ey, dd;
                if (ROWGATE) {
                    eg = (GATE == KDA_GATE_SCALAR) ? rowf[i] : 1.f;
                    ey = (GATE == KDA_GATE_SCALAR) ? rowi[i] : 1.f;
                    dd = dec_s[0];
                } else {
                    const float gm = pre[e] + g2[r][e];   // Gamma_i (log2), <= 0
                    eg = ex2(gm);
                    ey = ex2(-gm);
                    dd = dec[e];
                }
                kx[e] = kf[e] * eg;                    // K e^{Gamma}
                qx[e] = (qf[e] * p.scale) * eg;        // Q~ e^{Gamma}
                ky[e] = kf[e] * ey;                    // K e^{-Gamma}
                kd[e] = kf[e] * (dd * ey);             // K e^{Gamma_last - Gamma}
            }
            uint4 hi, lo;
            st_shared_v4(sm + M::KQ3, omn, pack8(kx));
            pack8_split(qx, hi, lo);
            st_shared_v4(sm + M::KQ3, omn + 16384, hi);
            st_shared_v4(sm + M::KQ3, omn + 32768, lo);
            pack8_split(ky, hi, lo);
            st_shared_v4(sm + M::KY, omn, hi);
            st_shared_v4(sm + M::KY, omn + 16384, lo);
            // Qg (rows 64-127 of the W|Qg image) and Kd go to the record as they are formed
            *reinterpret_cast<uint4*>(g_wq + omn + 16384) = pack8_f16(qx);
            *reinterpret_cast<uint4*>(g_kd + omn) = pack8_f16(kd);
        }
    } else if (!SLOW) {
        // ================= two references: row r_h = 32 h + 15 for the rows of half h, so
        // that each factor spans at most 16 rows of decay.  Columns j of half h take
        // 2^{G_rh - G_j} (rows 32 h .. 32 h + 31 of K e^{-G}'s space: hi, then lo); rows i
        // take 2^{G_i - G_rh} for h = 0 (every row) and h = 1 (rows of half 1).  The Gram
        // runs column half 1 first with the rows of half 1 over r_1, then column half 0
        // with those rows rebuilt over r_0, so rows 0-63 end as K 2^{G - G_r0}: the B
        // operand of W, whose columns are scaled by 2^{G_r0} when read out.  Rows of half
        // 1 park (G_i - G_r1, raw k, raw q) in tensor memory columns 192-255 meanwhile.
        const int hh = rg >> 3;   // warp-uniform: warps 4-7 hold the rows of half 1
        // per-channel terms come from shared memory row by row (register pressure):
        // G_r (gref_s row hh), 2^{G_r} (row 2 + hh), 2^{G_last - G_r} (row 4 + hh), and this
        // row group's prefix
        auto ld8 = [](const float* src, float (&d)[8]) {
            const float4 a = *reinterpret_cast<const float4*>(src), b = *reinterpret_cast<const float4*>(src + 4);
            d[0] = a.x; d[1] = a.y; d[2] = a.z; d[3] = a.w; d[4] = b.x; d[5] = b.y; d[6] = b.z; d[7] = b.w;
        };
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const uint32_t omn =
                basemn + (((uint32_t)(cq & 7) ^ (uint32_t)(4 * (rg & 1) + r)) << 4) + (uint32_t)(r * 128);
            float kf[8], qf[8], kx[8], qx[8], ky[8], t[8], dl[8], u[8];
            ld8(tot4 + rg * DK + c8, dl);
            ld8(gref_s + hh * DK + c8, u);
#pragma unroll
            for (int e = 0; e < 8; ++e) dl[e] = (dl[e] + g2[r][e]) - u[e];   // G_i - G_r
            if (hh) {   // parked for the rebuild over r_0: G_i - G_r1, raw k, raw q
                uint32_t park[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) park[e] = __float_as_uint(dl[e]);
                tmem_st8(tm + lane_base + 192u + 16u * r, park);
                park[0] = kraw[r].x; park[1] = kraw[r].y; park[2] = kraw[r].z; park[3] = kraw[r].w;
                park[4] = qraw[r].x; park[5] = qraw[r].y; park[6] = qraw[r].z; park[7] = qraw[r].w;
                tmem_st8(tm + lane_base + 200u + 16u * r, park);
            }
            unpack8(kraw[r], kf);
            unpack8(qraw[r], qf);
            dqp[r] = 0.f;
            ld8(gref_s + (4 + hh) * DK + c8, t);   // 2^{G_last - G_r}
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                dqp[r] = fmaf(kf[e], qf[e], dqp[r]);
                const float x = ex2(dl[e]), y = ex2(-dl[e]);
                qf[e] *= p.scale;
                kx[e] = kf[e] * x;
                qx[e] = qf[e] * x;
                ky[e] = kf[e] * y;
                // K e^{Gamma_last - Gamma}: where the first factor underflows, y <= 2^100 and the
                // dropped value is below 2^-26
                t[e] = kf[e] * (t[e] * y);
            }
            uint4 hi, lo;
            st_shared_v4(sm + M::KQ3, omn, pack8(kx));
            pack8_split(qx, hi, lo);
            st_shared_v4(sm + M::KQ3, omn + 16384, hi);
            st_shared_v4(sm + M::KQ3, omn + 32768, lo);
            pack8_split(ky, hi, lo);
            st_shared_v4(sm + M::KY, omn + 8192u * hh, hi);
            st_shared_v4(sm + M::KY, omn + 8192u * hh + 8192u, lo);
            *reinterpret_cast<uint4*>(g_kd + omn) = pack8_f16(t);
            ld8(gref_s + (2 + hh) * DK + c8, u);   // 2^{G_r}
#pragma unroll
            for (int e = 0; e < 8; ++e) t[e] = qx[e] * u[e];   // Q~ e^{Gamma}
            *reinterpret_cast<uint4*>(g_wq + omn + 16384) = pack8_f16(t);
        }
        if (hh) tmem_wait_st();
    } else {
        // ================= sub-block references
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
                Lr[e] = lv[e] - rv[e];         // Gamma_last - Gamma_r (log2)
            }
#pragma unroll
            for (int I = 1; I < 4; ++I) {
                if (I > b) {
                    const float4* ip = reinterpret_cast<const float4*>(gref_s + I * DK + c8);
                    const float4 i0 = ip[0], i1 = ip[1];
                    const float iv[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) z[I][e] = iv[e] - rv[e];   // Gamma_rI - Gamma_r (log2)
                }
            }
        }
        __syncthreads();   // the scan scratch shares region A with the j-side operands
        const uint32_t sw0 = (uint32_t)(cq & 7);
        // the same rows inside a 128-row K-major tile: K-atom stride 16 KB
        const uint32_t baseY = (uint32_t)((cq >> 3) * 16384 + (rg >> 1) * 1024 + (rg & 1) * 512);
        const uint32_t base128 = (uint32_t)((cq >> 3) * 16384 + ((rg >> 1) + 2 * b) * 1024 + (rg & 1) * 512);
        // Q~ i-side lo rows: row i of a 64-row K-major tile (K-atom stride 8 KB)
        const uint32_t base64 = (uint32_t)((cq >> 3) * 8192 + (rg >> 1) * 1024 + (rg & 1) * 512);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const uint32_t swz = ((sw0 ^ (uint32_t)(4 * (rg & 1) + r)) << 4) + (uint32_t)(r * 128);
            const uint32_t o128 = base128 + swz, omn = basemn + swz;
            const uint32_t oy = baseY + swz;   // + (I >> 1) * 32768 + (I & 1) * 8192 for version I
            float kf[8], qf[8], x[8], y[8], t[8], dl[8];
            unpack8(kraw[r], kf);
            unpack8(qraw[r], qf);
            dqp[r] = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                dqp[r] = fmaf(kf[e], qf[e], dqp[r]);
                dl[e] = (pre[e] + g2[r][e]) - gr[e];   // Gamma_i - Gamma_r (log2)
                x[e] = ex2(dl[e]);
                y[e] = ex2(-dl[e]);
                qf[e] *= p.scale;
            }
            uint4 hi, lo;
            // Gram i-side: K rows at 32 b + (i - 16 b), Q rows 16 further (hi); Q lo rows at i
#pragma unroll
            for (int e = 0; e < 8; ++e) t[e] = kf[e] * x[e];
            st_shared_v4(sm + M::OX, o128, pack8(t));
#pragma unroll
            for (int e = 0; e < 8; ++e) t[e] = qf[e] * x[e];
            pack8_split(t, hi, lo);
            st_shared_v4(sm + M::OX, o128 + 2048, hi);
            st_shared_v4(sm + M::OXL, base64 + swz, lo);
            // Gram j-side for this sub-block and the later ones (hi and lo); a later
            // sub-block I's factor 2^{Gamma_rI - Gamma_j} <= 1 is one power, not the product
            // of 2^{Gamma_r - Gamma_j} and 2^{Gamma_rI - Gamma_r}: the second can underflow
            // where the product does not
            float ky[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) ky[e] = kf[e] * y[e];
            pack8_split(ky, hi, lo);
            st_shared_v4(sm + M::OY + (b >> 1) * 32768 + (b & 1) * 8192, oy, hi);
            st_shared_v4(sm + M::OYL + (b >> 1) * 32768 + (b & 1) * 8192, oy, lo);
#pragma unroll
            for (int I = 1; I < 4; ++I) {
                if (I > b) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) t[e] = kf[e] * ex2(z[I][e] - dl[e]);
                    pack8_split(t, hi, lo);
                    st_shared_v4(sm + M::OY + (I >> 1) * 32768 + (I & 1) * 8192, oy, hi);
                    st_shared_v4(sm + M::OYL + (I >> 1) * 32768 + (I & 1) * 8192, oy, lo);
                }
            }
            // K e^Gamma (shared, MN-major), Q~ e^Gamma and K e^{Gamma_last - Gamma} (record)
            float t2[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float eg = Er[e] * x[e];
                t[e] = kf[e] * eg;
                t2[e] = qf[e] * eg;
            }
            st_shared_v4(sm + M::KG, omn, pack8(t));
            *reinterpret_cast<uint4*>(g_wq + omn + 16384) = pack8_f16(t2);
#pragma unroll
            for (int e = 0; e < 8; ++e) t[e] = kf[e] * ex2(Lr[e] - dl[e]);   // one power, as above
            *reinterpret_cast<uint4*>(g_kd + omn) = pack8_f16(t);
        }
    }
    store_dq();
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ================= Gram MMAs (hi * hi + hi * lo + lo * hi, fp32 accumulation)
    // one reference: cols 0-127 = [K e^G ; Q~ e^G]_n . [(K e^-G) hi ; (K e^-G) lo]_j
    // (M = 128, N = 128: the two j-side terms side by side), cols 128-191 =
    // [Q~ e^G (hi) ; Q~ e^G (lo)]_n . (K e^-G)_j (hi) (N = 64): lanes 64-127 of it are the
    // lo * hi term of the Qp rows
    // sub-blocks: group g (M = 128, N = 64): A rows 0-63 are the j-side of version 2g,
    // rows 64-127 that of version 2g+1 (hi, then lo); B rows the i-side rows of sub-blocks
    // 2g, 2g+1; cols 128 + 32 g: the same j-side (hi) against their Q~ lo rows (N = 32)
    // two references: per column half h, cols 96 h + (0-31 hi, 32-63 lo) = the same
    // products against the 32 j-side rows of half h, cols 96 h + 64 the lo * hi term
    auto gram_half = [&](int h) {
        const uint32_t kq = sbase + M::KQ3, ky = sbase + M::KY + 16384u * h;
#pragma unroll
        for (int s8 = 0; s8 < 8; ++s8)
            mma_bf16(tm + TM_GRAM + 96 * h, rowview_desc(kq, s8), rowview_desc(ky, s8),
                     idesc_bf16(128, 64, false, false), s8 > 0);
#pragma unroll
        for (int s8 = 0; s8 < 8; ++s8)
            mma_bf16(tm + TM_GRAM + 96 * h + 64, rowview_desc(kq + 16384, s8), rowview_desc(ky, s8),
                     idesc_bf16(128, 32, false, false), s8 > 0);
        mma_commit(mma_bar);
    };
    if (!SLOW && two) {
        if (tid == 0) gram_half(1);
        if (!wait_all(mma_bar, mma_phase)) return 2;
        tc_fence_after();
        if (rg >= 8) {   // rows of half 1: the i-side over r_0 for column half 0
            float d10[8];
            {
                const float4* a = reinterpret_cast<const float4*>(gref_s + c8);
                const float4* b = reinterpret_cast<const float4*>(gref_s + DK + c8);
                const float4 a0 = a[0], a1 = a[1], b0 = b[0], b1 = b[1];
                d10[0] = b0.x - a0.x; d10[1] = b0.y - a0.y; d10[2] = b0.z - a0.z; d10[3] = b0.w - a0.w;
                d10[4] = b1.x - a1.x; d10[5] = b1.y - a1.y; d10[6] = b1.z - a1.z; d10[7] = b1.w - a1.w;
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const uint32_t omn =
                    basemn + (((uint32_t)(cq & 7) ^ (uint32_t)(4 * (rg & 1) + r)) << 4) + (uint32_t)(r * 128);
                float park[16], kf[8], qf[8], kx[8], qx[8];
                tmem_ld16(tm + lane_base + 192u + 16u * r, park);
                const uint4 kr4 = make_uint4(__float_as_uint(park[8]), __float_as_uint(park[9]),
                                             __float_as_uint(park[10]), __float_as_uint(park[11]));
                const uint4 qr4 = make_uint4(__float_as_uint(park[12]), __float_as_uint(park[13]),
                                             __float_as_uint(park[14]), __float_as_uint(park[15]));
                unpack8(kr4, kf);
                unpack8(qr4, qf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float x = ex2(park[e] + d10[e]);   // 2^{G_i - G_r0} <= 1
                    kx[e] = kf[e] * x;
                    qx[e] = (qf[e] * p.scale) * x;
                }
                uint4 hi, lo;
                st_shared_v4(sm + M::KQ3, omn, pack8(kx));
                pack8_split(qx, hi, lo);
                st_shared_v4(sm + M::KQ3, omn + 16384, hi);
                st_shared_v4(sm + M::KQ3, omn + 32768, lo);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) gram_half(0);
    }
    if (tid == 0 && !(!SLOW && two)) {
        if (!SLOW) {
            const uint32_t kq = sbase + M::KQ3, ky = sbase + M::KY;
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8)
                mma_bf16(tm + TM_GRAM, rowview_desc(kq, s8), rowview_desc(ky, s8),
                         idesc_bf16(128, 128, false, false), s8 > 0);
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8)
                mma_bf16(tm + TM_GRAM + 128, rowview_desc(kq + 16384, s8), rowview_desc(ky, s8),
                         idesc_bf16(128, 64, false, false), s8 > 0);
        } else {
            const uint32_t ox = sbase + M::OX, oxl = sbase + M::OXL, oy = sbase + M::OY, oyl = sbase + M::OYL;
#pragma unroll
            for (int g = 0; g < 2; ++g) {
#pragma unroll
                for (int s8 = 0; s8 < 8; ++s8)
                    mma_bf16(tm + TM_GRAM + 64 * g, kmaj_desc(oy + g * 32768, 128, s8),
                             kmaj_desc(ox + g * 8192, 128, s8), idesc_bf16(128, 64, false, false), s8 > 0);
#pragma unroll
                for (int s8 = 0; s8 < 8; ++s8)
                    mma_bf16(tm + TM_GRAM + 128 + 32 * g, kmaj_desc(oy + g * 32768, 128, s8),
                             kmaj_desc(oxl + g * 4096, 64, s8), idesc_bf16(128, 32, false, false), s8 > 0);
#pragma unroll
                for (int s8 = 0; s8 < 8; ++s8)
                    mma_bf16(tm + TM_GRAM + 64 * g, kmaj_desc(oyl + g * 32768, 128, s8),
                             kmaj_desc(ox + g * 8192, 128, s8), idesc_bf16(128, 64, false, false), 1);
            }
        }
        mma_commit(mma_bar);
    }
    if (!wait_all(mma_bar, mma_phase)) return 2;
    tc_fence_after();
    // ================= coupling matrix L (fp32, shared) and lower(Qp) (fp16, record)
    float* Lm = reinterpret_cast<float*>(sm + M::L);
    float* TF = reinterpret_cast<float*>(sm + M::TF);
    if (!SLOW) {
        // lane n = 32 sp + lane: row i of P (n < 64) or of Qp (n >= 64); columns 32 half ..
        // (two references: lanes of rows outside column half 1's row range hold values of
        // no meaning there, all above the diagonal and masked by selection)
        const int n = 32 * sp + lane, j0 = 32 * half;
        const bool tw = two_ref();
        const uint32_t chh = tw ? 96u * half : (uint32_t)j0;              // hi * hi
        const uint32_t chl = tw ? chh + 32u : 64u + j0;                    // hi * lo
        const uint32_t clh = tw ? chh + 64u : 128u + j0;                   // lo * hi
        float v[32];
        {
            float w[32];
            tmem_ld32(tm + lane_base + TM_GRAM + chh, v);
            tmem_ld32(tm + lane_base + TM_GRAM + chl, w);   // the hi * lo term
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] += w[e];
        }
        if (n < 64) {   // warp-uniform (sub-partitions 0-1)
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
            float w[32];
            tmem_ld32(tm + lane_base + TM_GRAM + clh, w);   // the lo * hi term
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float t8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int j = j0 + 8 * q + e;
                    t8[e] = (j < i) ? v[8 * q + e] + w[8 * q + e] : ((j == i) ? dii : 0.f);
                }
                st_shared_v4(sm + M::AQST, kmaj_off(i, j0 + 8 * q, 64), pack8_f16(t8));
            }
        }
    } else {
        // warp group g reads Gram group g; lanes of sub-partitions 0-1 hold rows j of
        // sub-block 2g's version, those of 2-3 rows j of sub-block 2g+1's version
        const int g = half, hi = sp >> 1;
        const int I = 2 * g + hi, j = 32 * (sp & 1) + lane;
        __half* aqs = reinterpret_cast<__half*>(sm + M::AQST);
        float v[32], w[16];
        tmem_ld32(tm + lane_base + TM_GRAM + 64 * g + 32 * hi, v);
        tmem_ld16(tm + lane_base + TM_GRAM + 128 + 32 * g + 16 * hi, w);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int i = 16 * I + u;
            Lm[i * LDT + j] = (j < i) ? beta_s[i] * v[u] : 0.f;
            aqs[kmaj_off(i, j, 64) >> 1] =
                __float2half_rn((j < i) ? v[16 + u] + w[u] : ((j == i) ? dq_s[i] : 0.f));
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {   // the staged lower(Qp) tile to the record
        bulk_store(rec_p + rec::AQ, sm + M::AQST, 8192u);
        bulk_commit();
    }
    // ================= T = (I + L)^{-1}: diagonal 16x16 blocks by forward substitution
    // (lane = column), then the off-diagonal blocks
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
    }
    if (tid == 0) bulk_wait_read();   // the staging is overwritten from here on
    __syncthreads();
    offdiag_columns(TF, Lm, reinterpret_cast<float*>(sm + M::NS), warp, lane);
    // T diag(beta) -> two-term bf16 expansion (K-major, K = j), 8 columns per step
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
        uint4 hi, lo;
        pack8_split(t8, hi, lo);
        st_shared_v4(sm + M::TB, kmaj_off(i, j0, 64), hi);
        st_shared_v4(sm + M::TBL, kmaj_off(i, j0, 64), lo);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ================= W = T diag(beta) K e^G (M = 64, N = 128: lanes 0-15 of each
    // sub-partition), over both terms of T diag(beta), and U^T = V^T [hi ; lo]^T
    // (M = 128 over the value index, N = 128: the two terms side by side)
    wait_v();   // V landed long ago; every thread observes it before its tiles are MMA operands
    if (tid == 0) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const uint32_t tb = sbase + (t == 0 ? M::TB : M::TBL);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_bf16(tm + TM_W, kmaj_desc(tb, 64, s), mnmaj_desc(sbase + M::KG, 128, s),
                         idesc_bf16(64, 128, false, true), t > 0 || s > 0);
        }
        // V: the two 64-column TMA tiles are the MN halves (8 KB apart) of one MN-major
        // operand; k-step s covers tokens 16 s .. 16 s + 15
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_bf16(tm + TM_UT, desc_sw128(sbase + M::RV + 2048u * s, 8192u, 1024u),
                     kmaj_desc(sbase + M::TB, 128, s), idesc_bf16(128, 128, true, false), s > 0);
        mma_commit(mma_bar);
    }
    if (!wait_all(mma_bar, mma_phase)) return 2;
    tc_fence_after();
    {
        // W: lane l < 16 of each sub-partition holds row 16 sp + l; columns 64 half ..
        const int i = 16 * sp + (lane & 15);
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
            float v[32];
            tmem_ld32(tm + lane_base + TM_W + 64 * half + 32 * hc, v);
            if (lane < 16) {
                // two references: W's columns take 2^{G_r0} (K e^G = (K 2^{G - G_r0}) 2^{G_r0})
                const float4* f = reinterpret_cast<const float4*>(gref_s + 2 * DK + 64 * half + 32 * hc);
                const bool tw = two_ref();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (tw) {
                        const float4 s0 = f[2 * q], s1 = f[2 * q + 1];
                        v[8 * q] *= s0.x;
                        v[8 * q + 1] *= s0.y;
                        v[8 * q + 2] *= s0.z;
                        v[8 * q + 3] *= s0.w;
                        v[8 * q + 4] *= s1.x;
                        v[8 * q + 5] *= s1.y;
                        v[8 * q + 6] *= s1.z;
                        v[8 * q + 7] *= s1.w;
                    }
                    st_shared_v4(sm + M::WST, mnmaj_off(64 * half + 32 * hc + 8 * q, i, 128), pack8_f16(v + 8 * q));
                }
            }
        }
        // U^T: lane = value row v, columns (tokens) 32 half .., hi term + lo term
        const int vr = 32 * sp + lane;
        float u[32], ul[32];
        tmem_ld32(tm + lane_base + TM_UT + 32 * half, u);
        tmem_ld32(tm + lane_base + TM_UT + 64 + 32 * half, ul);
#pragma unroll
        for (int e = 0; e < 32; ++e) u[e] += ul[e];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            st_shared_v4(sm + M::UST, kmaj_off(vr, 32 * half + 8 * q, 128), pack8_f16(u + 8 * q));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {   // W (rows 0-63 of the W|Qg image) and U^T
        bulk_store(rec_p + rec::WQ, sm + M::WST, 16384u);
        bulk_store(rec_p + rec::UT, sm + M::UST, 16384u);
        bulk_commit();
        bulk_wait_read();
    }
    __syncthreads();
    return 0;
}

template <int GATE, bool SLOW>
__global__ void __launch_bounds__(NT, SLOW ? 1 : 2) kda_chunk_wy_kernel(const __grid_constant__ WyParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    using M = WyMap<SLOW>;
    const int tid = threadIdx.x, warp = tid >> 5;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(sm + M::BAR);
    uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(full_bar + 2);
    int* flag_s = reinterpret_cast<int*>(full_bar + 3);
    pdl_launch_dependents();
    if (SLOW) pdl_wait();   // the list is complete once the one-reference kernel is
    const int count = SLOW ? *p.slow : 0;
    if (SLOW && (int)blockIdx.x >= count) return;
    if (tid == 0) {
        mbar_init(full_bar, 1);
        mbar_init(full_bar + 1, 1);
        mbar_init(full_bar + 4, 1);
        *flag_s = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_base_s, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_base_s;
    uint32_t full_phase = 0, mma_phase = 0, v_phase = 0;
    if (!SLOW) {
        (void)wy_job<GATE, false>(p, sm, tm, blockIdx.x, blockIdx.y, full_phase, mma_phase, v_phase);
    } else {
        for (int x = blockIdx.x; x < count; x += gridDim.x) {
            const int job = p.slow[1 + x];
            if (wy_job<GATE, true>(p, sm, tm, job / p.H, job % p.H, full_phase, mma_phase, v_phase) == 2) break;
        }
    }
    if (tid == 0) bulk_wait_read();   // shared memory outlives no store that reads it
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, TMEM_COLS);
    }
}

// Chunk offsets of a packed batch: coff[n] = sum_{m < n} ceil(len_m / C), with
// inconsistent sequences counted as empty (and flagged, as everywhere else).
__global__ void __launch_bounds__(1024) kda_chunk_offsets_kernel(const int32_t* cu, int num_seqs, int T,
                                                                 int32_t* coff, int32_t* dev_status) {
    __shared__ int32_t warp_sums[32];
    __shared__ int32_t carry_s;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) carry_s = 0;
    __syncthreads();
    for (int base = 0; base < num_seqs; base += 1024) {
        const int n = base + tid;
        int cnt = 0;
        if (n < num_seqs) {
            const int a = cu[n], b = cu[n + 1];
            if (a < 0 || b < a || b > T || (n == 0 && a != 0)) {
                if (dev_status) atomicOr(dev_status, KDA_DEV_BAD_SEQLENS);
            } else {
                cnt = (b - a + C - 1) / C;
            }
        }
        int x = cnt;   // inclusive warp scan
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_sums[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int w = warp_sums[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            warp_sums[lane] = w;   // inclusive over warps
        }
        __syncthreads();
        const int carry = carry_s;
        const int excl = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + x - cnt;
        if (n < num_seqs) coff[n] = excl;
        __syncthreads();
        if (tid == 0) carry_s = carry + warp_sums[31];
        __syncthreads();
    }
    if (tid == 0) coff[num_seqs] = carry_s;
}

template <int GATE>
cudaError_t launch_wy_gate(const WyParams& p, long long slots, int sm_count, cudaStream_t st) {
    auto kf = kda_chunk_wy_kernel<GATE, false>;
    auto ks = kda_chunk_wy_kernel<GATE, true>;
    cudaError_t e = cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, wy_smem_bytes<false>());
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, wy_smem_bytes<true>());
    if (e != cudaSuccess) return e;
    // Prefetch distance: one CTA per SM, i.e. half of the two-per-SM resident wave.  It
    // measured best: a full wave ahead ran 1.3 % slower, prefetching nothing 2.6 %.
    WyParams pf = p;
    pf.ahead = sm_count;
    kf<<<dim3((unsigned)slots, (unsigned)p.H), NT, wy_smem_bytes<false>(), st>>>(pf);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // A quarter of the SMs: each of these CTAs (215 KB) holds its SM from the moment the
    // one-reference kernel drains from it, so the state scan launched behind this kernel
    // finds the other SMs free for its prologue while the one-reference kernel finishes.
    const long long jobs = slots * p.H;
    const int cap = sm_count / 4 > 0 ? sm_count / 4 : 1;
    const int grid = (int)(jobs < (long long)cap ? jobs : (long long)cap);
    return launch_after(ks, dim3(grid), NT, wy_smem_bytes<true>(), st, p);
}

}  // namespace

// The state-independent pass of the two-kernel prefill (see kda_chunk_record.cuh).
cudaError_t launch_chunk_wy(const ChunkArgs& a, uint8_t* ws, const rec::Layout& lay, cudaStream_t st) {
    WyParams p;
    memset(&p, 0, sizeof(p));
    p.g = a.g;
    p.beta = a.beta;
    p.cu_seqlens = a.cu_seqlens;
    p.dev_status = a.dev_status;
    p.slow = reinterpret_cast<int32_t*>(ws + lay.list_off);
    p.coff = a.cu_seqlens ? reinterpret_cast<const int32_t*>(ws + lay.coff_off) : nullptr;
    p.rec = ws + lay.rec_off;
    p.T = a.T;
    p.H = a.H;
    p.num_seqs = a.num_seqs;
    p.nc = (a.T + C - 1) / C;
    p.scale = a.scale;
    const long long tokens = (long long)a.B * a.T;
    if (tokens == 0 || lay.slots == 0) return cudaSuccess;
    p.group = a.H / a.Hk;
    bool ok = make_map(&p.map_k, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, a.Hk, tokens, DK, C,
                       CU_TENSOR_MAP_SWIZZLE_NONE) &&
              make_map(&p.map_q, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, a.Hk, tokens, DK, C,
                       CU_TENSOR_MAP_SWIZZLE_NONE) &&
              make_map(&p.map_v, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rec::DV, a.H, tokens, 64, C,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (ok && a.gate == KDA_GATE_CHANNEL)
        ok = make_map(&p.map_g, a.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, DK, a.H, tokens, DK, C,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(p.slow, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) return e;
    if (a.cu_seqlens) {
        kda_chunk_offsets_kernel<<<1, 1024, 0, st>>>(a.cu_seqlens, a.num_seqs, a.T,
                                                     const_cast<int32_t*>(p.coff), a.dev_status);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        (void)cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    switch (a.gate) {
        case KDA_GATE_CHANNEL: return launch_wy_gate<KDA_GATE_CHANNEL>(p, lay.slots, sms, st);
        case KDA_GATE_SCALAR: return launch_wy_gate<KDA_GATE_SCALAR>(p, lay.slots, sms, st);
        default: return launch_wy_gate<KDA_GATE_NONE>(p, lay.slots, sms, st);
    }
}

}  // namespace kda
