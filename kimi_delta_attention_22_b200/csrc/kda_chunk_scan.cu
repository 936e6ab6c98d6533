// kda_chunk_scan.cu -- the sequential half of the two-kernel tensor-core
// prefill: the inter-chunk state scan plus outputs, from the records the WY
// kernel wrote (layout and formulas in kda_chunk_record.cuh).
//
// One CTA per (sequence, head, value tile of BV columns) walks its sequence's
// chunks in order with the fp32 state tile S^T (128 x BV) in registers
// (thread = key channel, 32 value columns per group of four warps) and a bf16
// copy in shared memory as the MMA operand.  Per chunk, three groups of
// tcgen05 MMAs:
//
//   [W ; Qg] S^T          (M = 128, N = BV, K = 128)  -> E = U - W S^T  (lanes 0-63)
//   Kd^T E                (M = 128, N = BV, K = 64)   -> S^T <- Diag(dec) S^T + Kd^T E
//   [* ; Aqk] E  (accum.) (M = 128, N = BV, K = 64)   -> O = Qg S^T + Aqk E (lanes 64-127)
//
// Records stream in by bulk copy NSTAGE - 1 chunks ahead (L2 prefetch further
// ahead); the outputs of a chunk are read out while the next chunk's first MMA
// runs, so the dependent chain per chunk is MMA -> E -> MMA -> state update.
//
// Two schedules of that chunk step:
//
// * BV = 64 (two CTAs per (sequence, head), three record stages), used while
//   all CTAs fit in one wave: 8 state warps plus one MMA warp that holds no
//   state.  One thread of it issues every MMA and record copy, so no state
//   warp waits on MMA issue; the warps hand off through mbarriers only.
// * BV = 128 (one CTA, two stages), used when there are more CTAs than that:
//   16 state warps, one of whose threads also issues, with two CTA barriers
//   per chunk.  It reads each record once and issues the same number of MMAs
//   (an N = 128 MMA issues as fast as an N = 64 one), so it finishes more
//   chunks per SM.  A seventeenth warp would cap the registers at 96 and
//   spill.
#include "kda_chunk_record.cuh"
#include "kda_internal.cuh"
#include "kda_tc_common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;
using namespace tc;

constexpr int C = rec::C, DK = rec::DK, DV = rec::DV;
constexpr uint64_t kWaitNs = 1000000000ull;   // 1 s bound on every wait
constexpr int kAhead = 3;                      // records fetched into L2 this many chunks before their copy

template <int BV>
struct Cfg {
    static_assert(BV == 64 || BV == 128, "value tile of 64 or 128 columns");
    static constexpr bool MMA_WARP = BV == 64;  // schedule: dedicated MMA warp, or CTA barriers
    static constexpr int NW = BV / 8;           // state warps: 4 TMEM sub-partitions x BV / 32 value quarters
    static constexpr int NT = 32 * NW + (MMA_WARP ? 32 : 0);
    static constexpr int NVT = DV / BV;
    static constexpr int NSTAGE = (BV == 64) ? 3 : 2;
    // One stage = one chunk's record slice: W|Qg, Kd, Aqk, this tile's U (the
    // record's 64-column U tiles, back to back), dec.
    static constexpr int ST_WQ = 0, ST_KD = 32768, ST_AQ = 49152, ST_U = 57344;
    static constexpr int U_BYTES = 128 * BV;
    static constexpr int ST_DEC = ST_U + U_BYTES;
    static constexpr int STAGE = (ST_DEC + 512 + 1023) / 1024 * 1024;   // keeps operands 1 KB aligned
    static constexpr uint32_t STAGE_TX = 57344u + (uint32_t)U_BYTES + 512u;
    static constexpr int OFF_S = NSTAGE * STAGE;       // S^T bf16 (MN-major, MN = v, K = c)
    static constexpr int OFF_BAR = OFF_S + DK * BV * 2;   // full[NSTAGE], 7 barriers, tmem base, flag
    static constexpr int SMEM_BYTES = OFF_BAR + 128 + 1024;
    static constexpr uint32_t TMEM_COLS = (BV == 64) ? 256 : 512;
    static constexpr uint32_t TM_D1 = 0;                // 2 x BV columns by chunk parity: [W ; Qg] S^T, then O
    static constexpr uint32_t TM_DS = 2 * BV;           // Kd^T E
    static constexpr uint32_t kStage16 = STAGE >> 4;    // stage offset in descriptor units
    static constexpr uint32_t kS16 = 2 * BV;            // S k-step: 2 x 8 rows x BV x 2 B, in 16 B units
    static_assert(SMEM_BYTES <= 232448, "shared memory over the sm_100 per-block limit");
    static_assert(8 * (NSTAGE + 9) <= 128, "barrier block");
    static_assert(ST_AQ - ST_KD == 16384 && ST_U - ST_AQ == 8192, "the [* ; Aqk] window needs Kd|Aqk adjacent");
    static_assert(TM_DS + BV <= TMEM_COLS, "TMEM columns");
};

// Byte offset of U element (token row j, value v of the tile) in a stage: the
// record keeps U as 64-column MN-major tiles of 8 KB.
__device__ __forceinline__ uint32_t u_off(int v, int j) {
    return (uint32_t)(8192 * (v >> 6)) + mnmaj_off(v & 63, j, 64);
}

struct ScanParams {
    const uint8_t* rec;
    const int32_t* coff;
    const int32_t* cu_seqlens;
    const float* S0;
    float* S_T;
    __nv_bfloat16* out;
    int32_t* dev_status;
    int T, H, num_seqs, nc;
};

// What one CTA works on, and where its state threads sit.
template <int BV>
struct Tile {
    using G = Cfg<BV>;
    uint8_t* sm;
    uint32_t sbase, tm, lane_base;
    int h, vt, n, sp, vh, lane, c_own, v0;
    size_t sg;   // state offset of (n, h)

    // record copy of chunk m (slot first + m) into its stage
    __device__ __forceinline__ void load(const ScanParams& p, long long first, int m, uint64_t* full) const {
        uint8_t* dst = sm + (m % G::NSTAGE) * G::STAGE;
        const uint8_t* src = p.rec + ((size_t)(first + m) * p.H + h) * rec::BYTES;
        uint64_t* bar = full + (m % G::NSTAGE);
        mbar_arrive_expect_tx(bar, G::STAGE_TX);
        bulk_load(dst + G::ST_WQ, src + rec::WQ, 57344u, bar);
        bulk_load(dst + G::ST_U, src + rec::U + G::U_BYTES * vt, (uint32_t)G::U_BYTES, bar);
        bulk_load(dst + G::ST_DEC, src + rec::DEC, 512u, bar);
    }
    __device__ __forceinline__ void prefetch(const ScanParams& p, long long first, int m) const {
        const uint8_t* src = p.rec + ((size_t)(first + m) * p.H + h) * rec::BYTES;
        bulk_prefetch_l2(src + rec::WQ, 57344u);
        bulk_prefetch_l2(src + rec::U + G::U_BYTES * vt, (uint32_t)G::U_BYTES);
        bulk_prefetch_l2(src + rec::DEC, 512u);
    }

    // Operand descriptors of stage 0; k-step and stage offsets are added in 16-byte
    // units (every address stays below 256 KB, inside the 14-bit address field).
    __device__ __forceinline__ uint64_t d_wq() const { return rowview_desc(sbase + G::ST_WQ, 0); }
    __device__ __forceinline__ uint64_t d_s() const { return mnmaj_desc(sbase + G::OFF_S, BV, 0); }
    __device__ __forceinline__ uint64_t d_kd() const { return mnmaj_desc(sbase + G::ST_KD, 128, 0); }
    // U: 64-column MN-major tiles 8 KB apart (one tile when BV = 64)
    __device__ __forceinline__ uint64_t d_u() const {
        return desc_sw128(sbase + G::ST_U, BV == 64 ? 1024u : 8192u, 1024u);
    }
    __device__ __forceinline__ uint64_t d_aq() const { return kmaj_desc(sbase + G::ST_KD + 8192, 128, 0); }

    // [W ; Qg] S^T of chunk m into its parity's columns
    __device__ __forceinline__ void mma_ws(int m) const {
        const uint64_t so = (uint64_t)((m % G::NSTAGE) * G::kStage16), dWQ = d_wq(), dS = d_s();
#pragma unroll
        for (int s = 0; s < 8; ++s)
            mma_bf16(tm + G::TM_D1 + BV * (m & 1), dWQ + so + (uint64_t)((s >> 2) * 64 + (s & 3) * 2),
                     dS + (uint64_t)(s * G::kS16), idesc_bf16(128, BV, false, true), s > 0);
    }
    // Kd^T E of chunk m
    __device__ __forceinline__ void mma_kde(int m) const {
        const uint64_t so = (uint64_t)((m % G::NSTAGE) * G::kStage16), dKD = d_kd(), dU = d_u();
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_bf16(tm + G::TM_DS, dKD + so + (uint64_t)(s * 256), dU + so + (uint64_t)(s * 128),
                     idesc_bf16(128, BV, true, true), s > 0);
    }
    // [* ; Aqk] E of chunk m accumulated onto its [W ; Qg] S^T columns.  Rows 0-63
    // of the window are the second half of Kd: their products land in lanes 0-63,
    // which hold nothing that is read again.
    __device__ __forceinline__ void mma_aqe(int m) const {
        const uint64_t so = (uint64_t)((m % G::NSTAGE) * G::kStage16), dAQ = d_aq(), dU = d_u();
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_bf16(tm + G::TM_D1 + BV * (m & 1), dAQ + so + (uint64_t)(s * 2), dU + so + (uint64_t)(s * 128),
                     idesc_bf16(128, BV, false, true), 1);
    }

    // initial state of this thread's key channel and value columns, and its bf16 copy
    __device__ __forceinline__ void state_init(const ScanParams& p, float (&S)[32]) const {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int v = vt * BV + v0 + j;
            S[j] = p.S0 ? p.S0[sg + (size_t)v * DK + c_own] : 0.f;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) st_shared_v4(sm + G::OFF_S, mnmaj_off(v0 + 8 * q, c_own, BV), pack8(S + 8 * q));
        fence_async_smem();
    }
    // E = U - W S^T of chunk m in place over the stage's U tile (rows j = lanes 0-63)
    __device__ __forceinline__ void e_step(int m) const {
        uint8_t* stg = sm + (m % G::NSTAGE) * G::STAGE;
        const int j = 32 * sp + lane;
        float d[32];
        tmem_ld32(tm + lane_base + G::TM_D1 + BV * (m & 1) + 32 * vh, d);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t off = G::ST_U + u_off(v0 + 8 * q, j);
            float u[8];
            unpack8(*reinterpret_cast<const uint4*>(stg + off), u);
#pragma unroll
            for (int e = 0; e < 8; ++e) u[e] -= d[8 * q + e];
            st_shared_v4(stg, off, pack8(u));
        }
        fence_async_smem();
    }
    // S^T <- Diag(dec) S^T + Kd^T E (fp32 registers) and its bf16 operand copy
    __device__ __forceinline__ void s_step(int m, float (&S)[32]) const {
        const uint8_t* stg = sm + (m % G::NSTAGE) * G::STAGE;
        float ds[32];
        tmem_ld32(tm + lane_base + G::TM_DS + 32 * vh, ds);
        const float dec = reinterpret_cast<const float*>(stg + G::ST_DEC)[c_own];
#pragma unroll
        for (int jv = 0; jv < 32; ++jv) S[jv] = fmaf(S[jv], dec, ds[jv]);
#pragma unroll
        for (int q = 0; q < 4; ++q) st_shared_v4(sm + G::OFF_S, mnmaj_off(v0 + 8 * q, c_own, BV), pack8(S + 8 * q));
        fence_async_smem();
    }
    // outputs of chunk m (tokens cp .. cp + Lp - 1) from lanes 64-127 of its columns
    __device__ __forceinline__ void read_out(const ScanParams& p, int m, long long cp, int Lp) const {
        const int i = 32 * (sp - 2) + lane;
        float v[32];
        tmem_ld32(tm + lane_base + G::TM_D1 + BV * (m & 1) + 32 * vh, v);
        if (i < Lp) {
            __nv_bfloat16* op = p.out + ((size_t)(cp + i) * p.H + h) * DV + vt * BV + v0;
#pragma unroll
            for (int q = 0; q < 4; ++q) reinterpret_cast<uint4*>(op)[q] = pack8(v + 8 * q);
        }
    }
    __device__ __forceinline__ void state_store(const ScanParams& p, const float (&S)[32]) const {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int v = vt * BV + v0 + j;
            p.S_T[sg + (size_t)v * DK + c_own] = S[j];
        }
    }
};

// Bounded wait taken by every lane of a warp, with one verdict for the warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, kWaitNs));
}

// Barriers (one block after the record stages):
//   full[s]  record copy landed            (tx count; waited by the MMA thread)
//   bar1     [W ; Qg] S^T done             (commit)   -> E warps
//   bar2     Kd^T E done                   (commit)   -> state warps
//   bar3     [* ; Aqk] E accumulated       (commit)   -> output warps, stage reuse
//   eready   E tile stored                 (one arrival per E warp; MMA-warp schedule)
//   oread    outputs read out of TMEM      (one arrival per output warp; MMA-warp schedule)
//   sready   bf16 state copy stored        (one arrival per state warp; MMA-warp schedule)
//   drain    error path: completion of every MMA issued so far
// Each completes once per chunk, in chunk order, so chunk m's phase has parity
// m & 1; the handshakes keep each barrier at most one phase ahead of any
// thread that waits on it.
struct Bars {
    uint64_t *full, *bar1, *bar2, *bar3, *eready, *oread, *sready, *drain;
    uint32_t* tmem_base;
    volatile int* flag;
    template <int NSTAGE>
    __device__ __forceinline__ static Bars at(uint8_t* p) {
        Bars b;
        b.full = reinterpret_cast<uint64_t*>(p);
        b.bar1 = b.full + NSTAGE;
        b.bar2 = b.bar1 + 1;
        b.bar3 = b.bar1 + 2;
        b.eready = b.bar1 + 3;
        b.oread = b.bar1 + 4;
        b.sready = b.bar1 + 5;
        b.drain = b.bar1 + 6;
        b.tmem_base = reinterpret_cast<uint32_t*>(b.bar1 + 7);
        b.flag = reinterpret_cast<volatile int*>(b.bar1 + 8);
        return b;
    }
};

template <int BV>
__global__ void __launch_bounds__(Cfg<BV>::NT, 1) kda_chunk_scan_kernel(const __grid_constant__ ScanParams p) {
    using G = Cfg<BV>;
    constexpr int NSTAGE = G::NSTAGE, NW = G::NW;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    Tile<BV> t;
    t.sm = sm;
    t.sbase = smem_u32(sm);
    t.vt = blockIdx.x % G::NVT;
    t.h = (blockIdx.x / G::NVT) % p.H;
    t.n = blockIdx.x / (G::NVT * p.H);
    t.sp = warp & 3;                 // TMEM sub-partition
    t.vh = warp >> 2;                // 32-column value group
    t.lane = lane;
    t.lane_base = (uint32_t)(32 * t.sp) << 16;
    t.c_own = 32 * t.sp + lane;      // key channel of a state thread
    t.v0 = 32 * t.vh;
    t.sg = ((size_t)t.n * p.H + t.h) * DV * DK;
    const Bars b = Bars::at<NSTAGE>(sm + G::OFF_BAR);
    // MMA-warp schedule: warp NW issues; barrier schedule: thread 64 (warp 2, an
    // output warp, off the E path) issues besides its state work
    const bool state_thread = !G::MMA_WARP || warp < NW;
    const bool issuer = G::MMA_WARP ? tid == 32 * NW : tid == 64;

    long long bos, eos;
    if (!seq_bounds(p.cu_seqlens, t.n, p.T, p.num_seqs, p.dev_status, bos, eos)) return;
    const int nch = (int)((eos - bos + C - 1) / C);

    if (tid == 0) {
        for (int s = 0; s < NSTAGE; ++s) mbar_init(b.full + s, 1);
        mbar_init(b.bar1, 1);
        mbar_init(b.bar2, 1);
        mbar_init(b.bar3, 1);
        mbar_init(b.eready, NW / 2);
        mbar_init(b.oread, NW / 2);
        mbar_init(b.sready, NW);
        mbar_init(b.drain, 1);
        *b.flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(b.tmem_base, G::TMEM_COLS);
        tmem_relinquish();
    }
    __syncthreads();
    float S[32];
    if (state_thread) t.state_init(p, S);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    t.tm = *b.tmem_base;
    // everything above overlaps the tail of the WY kernels; records are read below
    pdl_wait();
    const long long first = p.cu_seqlens ? (long long)p.coff[t.n] : (long long)t.n * p.nc;
    int loaded = -1;   // issuer: last chunk whose record copy was issued
    int landed = 0;    // issuer: chunks below this one were seen complete on full[]
    if (issuer) {
        for (int m = 0; m < nch && m < NSTAGE - 1; ++m) t.load(p, first, m, b.full), loaded = m;
        for (int m = NSTAGE - 1; m < nch && m < NSTAGE - 1 + kAhead; ++m) t.prefetch(p, first, m);
    }
    // the stage of chunk m - 1 is refilled (chunk m + NSTAGE - 1) once its output MMAs are done
    auto refill = [&](int m) -> bool {
        if (m + NSTAGE - 1 < nch) {
            if (m > 0 && !mbar_wait(b.bar3, (uint32_t)((m - 1) & 1), kWaitNs)) return false;
            t.load(p, first, m + NSTAGE - 1, b.full);
            loaded = m + NSTAGE - 1;
        }
        if (m + NSTAGE - 1 + kAhead < nch) t.prefetch(p, first, m + NSTAGE - 1 + kAhead);
        return true;
    };

    long long c_prev = 0;
    int L_prev = 0;
    if constexpr (G::MMA_WARP) {
        if (warp == NW) {
            // ---- the MMA thread: waits and issues, nothing else
            if (lane == 0) {
                bool ok = nch == 0 || mbar_wait(b.full, 0, kWaitNs);
                if (ok && nch > 0) landed = 1;
                for (int m = 0; ok && m < nch; ++m) {
                    // state copy of chunk m - 1 stored (and its Kd^T E read out of TMEM)
                    if (m > 0 && !(ok = mbar_wait(b.sready, (uint32_t)((m - 1) & 1), kWaitNs))) break;
                    tc_fence_after();
                    t.mma_ws(m);
                    mma_commit(b.bar1);
                    if (!(ok = refill(m))) break;
                    if (!(ok = mbar_wait(b.eready, (uint32_t)(m & 1), kWaitNs))) break;
                    tc_fence_after();
                    t.mma_kde(m);
                    mma_commit(b.bar2);
                    // chunk m - 1's outputs are out of TMEM: its columns are free for chunk
                    // m + 1, and bar3 cannot run two phases ahead of the output warps
                    if (m > 0 && !(ok = mbar_wait(b.oread, (uint32_t)((m - 1) & 1), kWaitNs))) break;
                    tc_fence_after();
                    t.mma_aqe(m);
                    mma_commit(b.bar3);
                    if (m + 1 < nch) {
                        if (!(ok = mbar_wait(b.full + (m + 1) % NSTAGE, (uint32_t)(((m + 1) / NSTAGE) & 1),
                                             kWaitNs)))
                            break;
                        landed = m + 2;
                    }
                }
                if (!ok) *b.flag = 1;
            }
            __syncwarp();
        } else {
            // ---- state warps: E (sub-partitions 0-1) or outputs (2-3), then the state update
            bool ok = true;
            for (int m = 0; m < nch; ++m) {
                if (__any_sync(0xffffffffu, *b.flag != 0)) { ok = false; break; }
                const long long c0 = bos + (long long)m * C;
                const int L = (int)min((long long)C, eos - c0);
                if (t.sp >= 2) {
                    if (m > 0) {
                        if (!(ok = warp_wait(b.bar3, (uint32_t)((m - 1) & 1)))) break;
                        tc_fence_after();
                        t.read_out(p, m - 1, c_prev, L_prev);
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(b.oread);
                    }
                } else {
                    if (!(ok = warp_wait(b.bar1, (uint32_t)(m & 1)))) break;
                    tc_fence_after();
                    t.e_step(m);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(b.eready);
                }
                if (!(ok = warp_wait(b.bar2, (uint32_t)(m & 1)))) break;
                tc_fence_after();
                t.s_step(m, S);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(b.sready);
                c_prev = c0;
                L_prev = L;
            }
            if (ok && nch > 0 && t.sp >= 2) {
                if ((ok = warp_wait(b.bar3, (uint32_t)((nch - 1) & 1)))) {
                    tc_fence_after();
                    t.read_out(p, nch - 1, c_prev, L_prev);
                }
            }
            if (!ok && lane == 0) *b.flag = 1;
        }
        tc_fence_before();
        __syncthreads();
    } else {
        // ---- barrier schedule: two CTA barriers per chunk
        bool aborted = false;
        for (int m = 0; m < nch; ++m) {
            const long long c0 = bos + (long long)m * C;
            const int L = (int)min((long long)C, eos - c0);
            if (issuer) {
                if (!mbar_wait(b.full + m % NSTAGE, (uint32_t)((m / NSTAGE) & 1), kWaitNs)) *b.flag = 1;
                else landed = m + 1;
                tc_fence_after();
                t.mma_ws(m);
                mma_commit(b.bar1);
                if (!refill(m)) *b.flag = 1;
            }
            if (t.sp >= 2) {
                if (m > 0) {
                    if (!mbar_wait(b.bar3, (uint32_t)((m - 1) & 1), kWaitNs)) *b.flag = 1;
                    tc_fence_after();
                    t.read_out(p, m - 1, c_prev, L_prev);
                }
            } else {
                if (!mbar_wait(b.bar1, (uint32_t)(m & 1), kWaitNs)) *b.flag = 1;
                tc_fence_after();
                t.e_step(m);
            }
            tc_fence_before();
            __syncthreads();
            if (*b.flag != 0) { aborted = true; break; }
            if (issuer) {
                tc_fence_after();
                t.mma_kde(m);
                mma_commit(b.bar2);
                t.mma_aqe(m);
                mma_commit(b.bar3);
            }
            if (!mbar_wait(b.bar2, (uint32_t)(m & 1), kWaitNs)) *b.flag = 1;
            tc_fence_after();
            t.s_step(m, S);
            tc_fence_before();
            __syncthreads();
            if (*b.flag != 0) { aborted = true; break; }
            c_prev = c0;
            L_prev = L;
        }
        if (!aborted && nch > 0 && t.sp >= 2) {
            if (!mbar_wait(b.bar3, (uint32_t)((nch - 1) & 1), kWaitNs)) {
                *b.flag = 1;
            } else {
                tc_fence_after();
                t.read_out(p, nch - 1, c_prev, L_prev);
            }
        }
        __syncthreads();
    }
    if (*b.flag != 0) {
        if (p.dev_status && tid == 0) atomicOr(p.dev_status, KDA_DEV_TIMEOUT);
        // let copies / MMAs still in flight land before the memory goes away
        if (issuer) {
            mma_commit(b.drain);
            (void)mbar_wait(b.drain, 0, kWaitNs);
            for (int c = landed; c <= loaded; ++c)
                (void)mbar_wait(b.full + c % NSTAGE, (uint32_t)((c / NSTAGE) & 1), kWaitNs);
        }
    } else if (state_thread && p.S_T) {
        t.state_store(p, S);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(t.tm, G::TMEM_COLS);
    }
}

template <int BV>
cudaError_t launch_scan(const ScanParams& p, long long pairs, cudaStream_t st) {
    using G = Cfg<BV>;
    cudaError_t e = cudaFuncSetAttribute(kda_chunk_scan_kernel<BV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         G::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    return launch_after(kda_chunk_scan_kernel<BV>, dim3((unsigned)(pairs * G::NVT)), G::NT, G::SMEM_BYTES, st, p);
}

}  // namespace

cudaError_t launch_chunk_scan(const ChunkArgs& a, const uint8_t* ws, const rec::Layout& lay, cudaStream_t st) {
    ScanParams p;
    p.rec = ws + lay.rec_off;
    p.coff = a.cu_seqlens ? reinterpret_cast<const int32_t*>(ws + lay.coff_off) : nullptr;
    p.cu_seqlens = a.cu_seqlens;
    p.S0 = a.S0;
    p.S_T = a.S_T;
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.dev_status = a.dev_status;
    p.T = a.T;
    p.H = a.H;
    p.num_seqs = a.num_seqs;
    p.nc = (a.T + C - 1) / C;
    // 64-column tiles while they all fit in one wave (the chain per chunk is
    // shortest there); whole-width CTAs once there are more.
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long pairs = (long long)a.num_seqs * a.H;
    if (pairs * Cfg<64>::NVT <= sms) return launch_scan<64>(p, pairs, st);
    return launch_scan<128>(p, pairs, st);
}

}  // namespace kda
