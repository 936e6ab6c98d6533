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
// BV = 64 (two CTAs per (sequence, head), 256 threads, three record stages)
// has the shorter chain; BV = 128 (one CTA, 512 threads, two stages) reads each
// record once and issues the same number of MMAs (an N = 128 MMA issues as
// fast as an N = 64 one), so it finishes more chunks per SM when the CTAs do
// not all fit in one wave.
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
constexpr int kIss = 64;                       // warp 2 (an output warp, off the E path)

template <int BV>
struct Cfg {
    static_assert(BV == 64 || BV == 128, "value tile of 64 or 128 columns");
    static constexpr int NT = 4 * BV;          // 4 TMEM sub-partitions x BV / 32 value quarters
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
    static constexpr int OFF_BAR = OFF_S + DK * BV * 2;   // full[NSTAGE], mma1, ds, o2, tmem base, flag
    static constexpr int SMEM_BYTES = OFF_BAR + 128 + 1024;
    static constexpr uint32_t TMEM_COLS = (BV == 64) ? 256 : 512;
    static constexpr uint32_t TM_D1 = 0;                // 2 x BV columns by chunk parity: [W ; Qg] S^T, then O
    static constexpr uint32_t TM_DS = 2 * BV;           // Kd^T E
    static_assert(SMEM_BYTES <= 232448, "shared memory over the sm_100 per-block limit");
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

template <int BV>
__global__ void __launch_bounds__(Cfg<BV>::NT, 1) kda_chunk_scan_kernel(const __grid_constant__ ScanParams p) {
    using G = Cfg<BV>;
    constexpr int NVT = G::NVT, NSTAGE = G::NSTAGE, STAGE = G::STAGE;
    constexpr int ST_WQ = G::ST_WQ, ST_KD = G::ST_KD, ST_U = G::ST_U, ST_DEC = G::ST_DEC;
    constexpr int OFF_S = G::OFF_S, OFF_BAR = G::OFF_BAR;
    constexpr uint32_t TMEM_COLS = G::TMEM_COLS, TM_D1 = G::TM_D1, TM_DS = G::TM_DS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const int H = p.H;
    const int vt = blockIdx.x % NVT;
    const int h = (blockIdx.x / NVT) % H;
    const int n = blockIdx.x / (NVT * H);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sp = warp & 3, vh = warp >> 2;   // TMEM sub-partition, 32-column value group
    const uint32_t lane_base = (uint32_t)(32 * sp) << 16;
    const uint32_t sbase = smem_u32(sm);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint64_t* bar1 = full + NSTAGE;
    uint64_t* bar2 = bar1 + 1;
    uint64_t* bar3 = bar1 + 2;
    uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(bar1 + 3);
    volatile int* flag_s = reinterpret_cast<volatile int*>(bar1 + 4);
    uint64_t* drain = bar1 + 5;        // error path: completion of every MMA issued so far

    long long bos, eos;
    if (!seq_bounds(p.cu_seqlens, n, p.T, p.num_seqs, p.dev_status, bos, eos)) return;
    const int nch = (int)((eos - bos + C - 1) / C);

    if (tid == 0) {
        for (int s = 0; s < NSTAGE; ++s) mbar_init(full + s, 1);
        mbar_init(bar1, 1);
        mbar_init(bar2, 1);
        mbar_init(bar3, 1);
        mbar_init(drain, 1);
        *flag_s = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_base_s, TMEM_COLS);
        tmem_relinquish();
    }
    __syncthreads();

    long long first = 0;             // slot of the sequence's first chunk (set after pdl_wait)
    int loaded = -1;                 // last chunk whose record copy was issued (issuing thread)
    auto load_chunk = [&](int m) {   // issuing thread only
        loaded = m;
        uint8_t* dst = sm + (m % NSTAGE) * STAGE;
        const uint8_t* src = p.rec + ((size_t)(first + m) * H + h) * rec::BYTES;
        uint64_t* bar = full + (m % NSTAGE);
        mbar_arrive_expect_tx(bar, G::STAGE_TX);
        bulk_load(dst + ST_WQ, src + rec::WQ, 57344u, bar);
        bulk_load(dst + ST_U, src + rec::U + G::U_BYTES * vt, (uint32_t)G::U_BYTES, bar);
        bulk_load(dst + ST_DEC, src + rec::DEC, 512u, bar);
    };
    // ---- initial state: thread owns key channel c, value columns v0..v0+31
    const int c_own = 32 * sp + lane;
    const int v0 = 32 * vh;
    const size_t sg = ((size_t)n * H + h) * DV * DK;
    float S[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const int v = vt * BV + v0 + j;
        S[j] = p.S0 ? p.S0[sg + (size_t)v * DK + c_own] : 0.f;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) st_shared_v4(sm + OFF_S, mnmaj_off(v0 + 8 * q, c_own, BV), pack8(S + 8 * q));
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_base_s;
    // everything above overlaps the tail of the WY kernels; records are read below
    pdl_wait();
    first = p.cu_seqlens ? (long long)p.coff[n] : (long long)n * p.nc;
    constexpr int kAhead = 3;   // records fetched into L2 this many chunks before their copy
    auto prefetch_chunk = [&](int m) {
        const uint8_t* src = p.rec + ((size_t)(first + m) * H + h) * rec::BYTES;
        bulk_prefetch_l2(src + rec::WQ, 57344u);
        bulk_prefetch_l2(src + rec::U + G::U_BYTES * vt, (uint32_t)G::U_BYTES);
        bulk_prefetch_l2(src + rec::DEC, 512u);
    };
    if (tid == kIss) {
        for (int m = 0; m < nch && m < NSTAGE - 1; ++m) load_chunk(m);
        for (int m = NSTAGE - 1; m < nch && m < NSTAGE - 1 + kAhead; ++m) prefetch_chunk(m);
    }
    // Operand descriptors of stage 0; k-step and stage offsets are added in 16-byte
    // units (every address stays below 256 KB, inside the 14-bit address field).
    constexpr uint32_t kStage16 = STAGE >> 4;
    const uint64_t dWQ = rowview_desc(sbase + ST_WQ, 0);          // + (s/4)*64 + (s%4)*2
    constexpr uint32_t kS16 = 2 * BV;                              // S k-step: 2 x 8 rows x BV x 2 B
    const uint64_t dS = mnmaj_desc(sbase + OFF_S, BV, 0);          // + s*kS16
    const uint64_t dKD = mnmaj_desc(sbase + ST_KD, 128, 0);        // + s*256
    // U: 64-column MN-major tiles 8 KB apart (one tile when BV = 64); + s*128
    const uint64_t dU = desc_sw128(sbase + ST_U, BV == 64 ? 1024u : 8192u, 1024u);
    const uint64_t dAQ = kmaj_desc(sbase + ST_KD + 8192, 128, 0);  // + s*2

    // Outputs of chunk m (its O2 MMAs complete on bar3): rows live in lanes 64-127.
    auto read_out = [&](long long cp, int Lp, uint32_t col) {
        const int i = 32 * (sp - 2) + lane;
        float v[32];
        tmem_ld32(tm + lane_base + col + 32 * vh, v);
        if (i < Lp) {
            __nv_bfloat16* op = p.out + ((size_t)(cp + i) * H + h) * DV + vt * BV + v0;
#pragma unroll
            for (int q = 0; q < 4; ++q) reinterpret_cast<uint4*>(op)[q] = pack8(v + 8 * q);
        }
    };

    uint32_t ph1 = 0, ph2 = 0, ph3 = 0;
    bool aborted = false;
    int m_stop = 0;
    long long c_prev = 0;
    int L_prev = 0;
    for (int m = 0; m < nch; ++m) {
        const int st = m % NSTAGE, par = m & 1;
        const uint32_t full_ph = (uint32_t)((m / NSTAGE) & 1);
        uint8_t* stg = sm + st * STAGE;
        const long long c0 = bos + (long long)m * C;
        const int L = (int)min((long long)C, eos - c0);
        const uint32_t d1 = TM_D1 + BV * par;
        if (tid == kIss) {
            if (!mbar_wait(full + st, full_ph, kWaitNs)) *flag_s = 1;
            tc_fence_after();
            const uint64_t so = (uint64_t)(st * kStage16);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_bf16(tm + d1, dWQ + so + (uint64_t)((s >> 2) * 64 + (s & 3) * 2), dS + (uint64_t)(s * kS16),
                         idesc_bf16(128, BV, false, true), s > 0);
            mma_commit(bar1);
            // the stage of chunk m - 1 is free once its output MMAs are done
            if (m + NSTAGE - 1 < nch) {
                if (m > 0 && !mbar_wait(bar3, ph3, kWaitNs)) *flag_s = 1;
                load_chunk(m + NSTAGE - 1);
            }
            if (m + NSTAGE - 1 + kAhead < nch) prefetch_chunk(m + NSTAGE - 1 + kAhead);
        }
        if (sp >= 2) {
            if (m > 0) {
                if (!mbar_wait(bar3, ph3, kWaitNs)) *flag_s = 1;
                tc_fence_after();
                read_out(c_prev, L_prev, TM_D1 + BV * (par ^ 1));
            }
        } else {
            // E = U - W S^T over the U tile (same MN-major layout), rows j = lanes 0-63
            if (!mbar_wait(bar1, ph1, kWaitNs)) *flag_s = 1;
            tc_fence_after();
            const int j = 32 * sp + lane;
            float d[32];
            tmem_ld32(tm + lane_base + d1 + 32 * vh, d);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t off = ST_U + u_off(v0 + 8 * q, j);
                float u[8];
                unpack8(*reinterpret_cast<const uint4*>(stg + off), u);
#pragma unroll
                for (int e = 0; e < 8; ++e) u[e] -= d[8 * q + e];
                st_shared_v4(stg, off, pack8(u));
            }
            fence_async_smem();
        }
        if (m > 0) ph3 ^= 1u;
        ph1 ^= 1u;
        tc_fence_before();
        __syncthreads();
        if (*flag_s != 0) { aborted = true; m_stop = m; break; }
        if (tid == kIss) {
            tc_fence_after();
            const uint64_t so = (uint64_t)(st * kStage16);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_bf16(tm + TM_DS, dKD + so + (uint64_t)(s * 256), dU + so + (uint64_t)(s * 128),
                         idesc_bf16(128, BV, true, true), s > 0);
            mma_commit(bar2);
            // rows 0-63 of the window are the second half of Kd: their products land in
            // lanes 0-63, which hold nothing that is read again
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_bf16(tm + d1, dAQ + so + (uint64_t)(s * 2), dU + so + (uint64_t)(s * 128),
                         idesc_bf16(128, BV, false, true), 1);
            mma_commit(bar3);
        }
        // ---- S^T <- Diag(dec) S^T + Kd^T E (fp32 registers) and its bf16 operand copy
        if (!mbar_wait(bar2, ph2, kWaitNs)) *flag_s = 1;
        ph2 ^= 1u;
        tc_fence_after();
        {
            float ds[32];
            tmem_ld32(tm + lane_base + TM_DS + 32 * vh, ds);
            const float dec = reinterpret_cast<const float*>(stg + ST_DEC)[c_own];
#pragma unroll
            for (int jv = 0; jv < 32; ++jv) S[jv] = fmaf(S[jv], dec, ds[jv]);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                st_shared_v4(sm + OFF_S, mnmaj_off(v0 + 8 * q, c_own, BV), pack8(S + 8 * q));
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (*flag_s != 0) { aborted = true; m_stop = m; break; }
        c_prev = c0;
        L_prev = L;
    }
    if (!aborted && nch > 0) {
        if (sp >= 2) {
            if (!mbar_wait(bar3, ph3, kWaitNs)) {
                *flag_s = 1;
            } else {
                tc_fence_after();
                read_out(c_prev, L_prev, TM_D1 + BV * ((nch - 1) & 1));
            }
        }
        __syncthreads();
        aborted = *flag_s != 0;
        m_stop = nch;
    }
    if (aborted) {
        if (p.dev_status && tid == 0) atomicOr(p.dev_status, KDA_DEV_TIMEOUT);
        // let copies / MMAs still in flight land before the memory goes away
        if (tid == kIss) {
            mma_commit(drain);
            (void)mbar_wait(drain, 0, kWaitNs);
            for (int c = m_stop; c <= loaded; ++c)
                (void)mbar_wait(full + c % NSTAGE, (uint32_t)((c / NSTAGE) & 1), kWaitNs);
        }
    } else if (p.S_T) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int v = vt * BV + v0 + j;
            p.S_T[sg + (size_t)v * DK + c_own] = S[j];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, TMEM_COLS);
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
