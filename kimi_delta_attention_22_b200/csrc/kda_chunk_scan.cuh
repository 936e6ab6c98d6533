// kda_chunk_scan.cuh -- the sequential half of the two-kernel tensor-core
// prefill: the inter-chunk state scan plus outputs, from the records the WY
// kernel wrote (layout and formulas in kda_chunk_record.cuh).
//
// One CTA per (sequence, head) walks its sequence's chunks in order.  The
// state is held the way the pages write it, S (d_v x d_k) with one value row
// per tensor-memory lane, and it never leaves tensor memory: the fp32 S is the
// accumulator of E^T Kd, and its fp16 copy is the A operand of the next chunk's
// first product, read by the MMA straight from tensor memory, as is E^T.  Per
// chunk:
//
//   S [W ; Qg]^T   (M = 128, N = 128, K = 128)  -> E^T = U^T - S W^T (cols 0-63),
//                                                  S Qg^T (cols 64-127)
//   E^T Kd         (M = 128, N = 128, K = 64)   accumulated onto Diag(dec)-scaled S:
//                                                  S <- S Diag(dec) + E^T Kd
//   E^T Aqk^T      (M = 128, N = 64,  K = 64)   accumulated onto S Qg^T -> O^T
//
// The threads of value row v scale the fp32 S by dec ahead of time, while the
// first product runs, so the sequential chain of a chunk is: first product ->
// E^T -> E^T Kd -> fp16 copy of S.  Outputs are read out while the next chunk's
// first product runs.  Every tcgen05.mma costs its issuing thread tens of
// cycles, so the products are kept few and wide.
//
// One thread of a warp of its own issues every MMA, one thread of another every
// record copy; the state warps hand off through mbarriers only.  Every barrier completes once per chunk, in
// chunk order, so chunk m waits on parity m & 1, and each handshake keeps a
// barrier at most one phase ahead of any thread that waits on it (the waits and
// arrivals are listed at Bars below).
//
// Chunkwise form: GeekNews summary of "You could have come up with Kimi Delta
// Attention", section "Chunkwise KDA" (each chunk maps S_c to S_{c+1} plus the
// chunk's outputs).
#pragma once

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

template <int NW>
struct Cfg {
    static_assert(NW == 8 || NW == 16, "8 or 16 state warps");
    static constexpr int NPART = NW / 4;       // threads per value row (key-channel ranges)
    static constexpr int NT = 32 * NW + 64;    // state warps + the MMA warp + the copy warp
    static constexpr int SC = DK / NPART;      // state columns per thread
    static constexpr int EC = C / NPART;       // E^T / output columns (tokens) per thread
    static constexpr int NSTAGE = 2;
    static constexpr int STAGE = (rec::BYTES + 1023) / 1024 * 1024;   // operands stay 1 KB aligned
    // per-warp output staging: 32 value rows x EC tokens, bf16, token-major
    static constexpr int OUT_WARP = 32 * EC * 2;
    static constexpr int OFF_OUT = NSTAGE * STAGE;
    static constexpr int OFF_BAR = OFF_OUT + NW * OUT_WARP;
    static constexpr int SMEM_BYTES = OFF_BAR + 128 + 1024;
    static constexpr uint32_t TM_S = 0;      // 128 cols: fp32 S (accumulator of E^T Kd)
    static constexpr uint32_t TM_D1 = 128;   // 2 x 128 cols by chunk parity: S W^T | O^T
    static constexpr uint32_t TM_AS = 384;   // 64 cols: S as the fp16 A operand (K = key channel)
    static constexpr uint32_t TM_AE = 448;   // 32 cols: E^T as the fp16 A operand (K = token)
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(SMEM_BYTES <= 232448, "shared memory over the sm_100 per-block limit");
    static_assert(8 * (2 * NSTAGE + 9) <= 128, "barrier block");
};

struct ScanParams {
    const uint8_t* rec;
    const int32_t* coff;
    const int32_t* cu_seqlens;
    const float* S0;
    float* S_T;
    __nv_bfloat16* out;   // null: outputs not written (state checkpoints only)
    float* S_chk;         // null, or [slot][H][d_v][d_k]: the incoming state of every chunk
    int32_t* dev_status;
    int T, H, num_seqs, nc;
};

// TMEM load of N consecutive fp32 columns (N = 16, 32 or 64) into v, one wait.
template <int N>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, float* v) {
    if constexpr (N == 16) {
        tmem_ld16(taddr, v);
    } else if constexpr (N == 32) {
        tmem_ld32(taddr, v);
    } else {
        tmem_ld64(taddr, v);
    }
}
// TMEM store of N consecutive 32-bit columns (N = 8, 16 or 32), no wait.
template <int N>
__device__ __forceinline__ void tmem_st_n(uint32_t taddr, const uint32_t* r) {
    if constexpr (N == 8) {
        tmem_st8(taddr, r);
    } else if constexpr (N == 16) {
        tmem_st16(taddr, r);
    } else {
        tmem_st32(taddr, r);
    }
}

// What one CTA works on, and where its thread sits.
template <int NW>
struct Tile {
    using G = Cfg<NW>;
    uint8_t* sm;
    uint32_t sbase, tm, lane_base;
    int h, n, v, part;
    size_t sg;   // state offset of (n, h)

    // record copy of chunk m (slot first + m) into its stage: one bulk copy
    __device__ __forceinline__ void load(const ScanParams& p, long long first, int m, uint64_t* full) const {
        uint64_t* bar = full + (m % G::NSTAGE);
        mbar_arrive_expect_tx(bar, (uint32_t)rec::BYTES);
        bulk_load(sm + (m % G::NSTAGE) * G::STAGE, p.rec + ((size_t)(first + m) * p.H + h) * rec::BYTES,
                  (uint32_t)rec::BYTES, bar);
    }
    __device__ __forceinline__ void prefetch(const ScanParams& p, long long first, int m) const {
        bulk_prefetch_l2(p.rec + ((size_t)(first + m) * p.H + h) * rec::BYTES, (uint32_t)rec::BYTES);
    }

    // S_m [W ; Qg]^T of chunk m into its parity's D1 columns
    __device__ __forceinline__ void mma1(int m) const {
        const uint32_t st = sbase + (uint32_t)((m % G::NSTAGE) * G::STAGE);
#pragma unroll
        for (int s = 0; s < 8; ++s)
            mma_tmem_a(tm + G::TM_D1 + 128u * (uint32_t)(m & 1), tm + G::TM_AS + 8u * s,
                       rowview_desc(st + rec::WQ, s), idesc_f16(128, 128, false, false), s > 0);
    }
    // E^T Kd of chunk m accumulated onto the Diag(dec)-scaled fp32 S
    __device__ __forceinline__ void mma2(int m) const {
        const uint32_t st = sbase + (uint32_t)((m % G::NSTAGE) * G::STAGE);
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_tmem_a(tm + G::TM_S, tm + G::TM_AE + 8u * s, mnmaj_desc(st + rec::KD, 128, s),
                       idesc_f16(128, 128, false, true), 1);
    }
    // E^T Aqk^T of chunk m accumulated onto its S Qg^T columns
    __device__ __forceinline__ void mma3(int m) const {
        const uint32_t st = sbase + (uint32_t)((m % G::NSTAGE) * G::STAGE);
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_tmem_a(tm + G::TM_D1 + 128u * (uint32_t)(m & 1) + 64u, tm + G::TM_AE + 8u * s,
                       kmaj_desc(st + rec::AQ, 64, s), idesc_f16(128, 64, false, false), 1);
    }

    // initial fp32 state of this thread's row slice and its fp16 copy
    __device__ __forceinline__ void state_init(const ScanParams& p) const {
        const float* src = p.S0 ? p.S0 + sg + (size_t)v * DK + G::SC * part : nullptr;
#pragma unroll
        for (int c32 = 0; c32 < G::SC / 32; ++c32) {
            uint32_t x[32], r[16];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 f = src ? reinterpret_cast<const float4*>(src)[8 * c32 + q]
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                x[4 * q] = __float_as_uint(f.x); x[4 * q + 1] = __float_as_uint(f.y);
                x[4 * q + 2] = __float_as_uint(f.z); x[4 * q + 3] = __float_as_uint(f.w);
                r[2 * q] = pack_f16(f.x, f.y);
                r[2 * q + 1] = pack_f16(f.z, f.w);
            }
            tmem_st32(tm + lane_base + G::TM_S + G::SC * part + 32 * c32, x);
            tmem_st16(tm + lane_base + G::TM_AS + (G::SC / 2) * part + 16 * c32, r);
        }
        tmem_wait_st();
    }
    // this thread's slice of U^T of chunk m (read before S W^T completes)
    __device__ __forceinline__ void load_ut(int m, uint4 (&u)[G::EC / 8]) const {
        const uint8_t* stg = sm + (m % G::NSTAGE) * G::STAGE;
#pragma unroll
        for (int q = 0; q < G::EC / 8; ++q)
            u[q] = *reinterpret_cast<const uint4*>(stg + rec::UT + kmaj_off(v, G::EC * part + 8 * q, 128));
    }
    // S <- S Diag(dec of chunk m), ahead of the accumulation of E^T Kd; S (the incoming
    // state of chunk m, this thread's SC columns of row v) is also left in keep
    __device__ __forceinline__ void decay(int m, float (&keep)[G::SC]) const {
        const float4* dec = reinterpret_cast<const float4*>(sm + (m % G::NSTAGE) * G::STAGE + rec::DEC) +
                            (G::SC / 4) * part;
#pragma unroll
        for (int c32 = 0; c32 < G::SC / 32; ++c32) {
            float* x = keep + 32 * c32;
            tmem_ld32(tm + lane_base + G::TM_S + G::SC * part + 32 * c32, x);
            uint32_t r[32];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 g = dec[8 * c32 + q];
                r[4 * q] = __float_as_uint(x[4 * q] * g.x);
                r[4 * q + 1] = __float_as_uint(x[4 * q + 1] * g.y);
                r[4 * q + 2] = __float_as_uint(x[4 * q + 2] * g.z);
                r[4 * q + 3] = __float_as_uint(x[4 * q + 3] * g.w);
            }
            tmem_st32(tm + lane_base + G::TM_S + G::SC * part + 32 * c32, r);
        }
        tmem_wait_st();
    }
    // E^T = U^T - S W^T of chunk m (this thread's tokens), as the A operand
    __device__ __forceinline__ void e_step(int m, const uint4 (&ut)[G::EC / 8]) const {
        float d[G::EC];
        tmem_ld_n<G::EC>(tm + lane_base + G::TM_D1 + 128u * (uint32_t)(m & 1) + G::EC * part, d);
        uint32_t r[G::EC / 2];
#pragma unroll
        for (int q = 0; q < G::EC / 8; ++q) {
            float u[8];
            unpack8_f16(ut[q], u);
#pragma unroll
            for (int e = 0; e < 4; ++e)
                r[4 * q + e] = pack_f16(u[2 * e] - d[8 * q + 2 * e], u[2 * e + 1] - d[8 * q + 2 * e + 1]);
        }
        tmem_st_n<G::EC / 2>(tm + lane_base + G::TM_AE + (G::EC / 2) * part, r);
        tmem_wait_st();
    }
    // the fp16 copy of the updated S (the next chunk's A operand)
    __device__ __forceinline__ void s_copy() const {
#pragma unroll
        for (int c32 = 0; c32 < G::SC / 32; ++c32) {
            float x[32];
            tmem_ld32(tm + lane_base + G::TM_S + G::SC * part + 32 * c32, x);
            uint32_t r[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = pack_f16(x[2 * i], x[2 * i + 1]);
            tmem_st16(tm + lane_base + G::TM_AS + (G::SC / 2) * part + 16 * c32, r);
        }
        tmem_wait_st();
    }
    // outputs of chunk m (tokens c0 .. c0 + L - 1): this thread's value row over its EC
    // tokens goes token-major into the warp's staging block (one 64-byte row of 32 values
    // per token), which the warp then writes out as 16-byte vectors
    __device__ __forceinline__ void read_out(const ScanParams& p, int m, long long c0, int L, int warp) const {
        if (p.out == nullptr) return;
        float o[G::EC];
        tmem_ld_n<G::EC>(tm + lane_base + G::TM_D1 + 128u * (uint32_t)(m & 1) + 64u + G::EC * part, o);
        __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(sm + G::OFF_OUT + warp * G::OUT_WARP);
        const int lane = v & 31;
#pragma unroll
        for (int i = 0; i < G::EC; ++i) stg[32 * i + lane] = __float2bfloat16_rn(o[i]);
        __syncwarp();
        const size_t tstride = (size_t)p.H * DV;
        __nv_bfloat16* op = p.out + ((size_t)c0 * p.H + h) * DV + (v - lane);
#pragma unroll
        for (int r = 0; r < G::EC / 8; ++r) {
            const int q = lane + 32 * r, i = q >> 2, cc = q & 3;   // token i, 8-value chunk cc
            const int tok = G::EC * part + i;
            const uint4 x = *reinterpret_cast<const uint4*>(stg + 32 * i + 8 * cc);
            if (tok < L) *reinterpret_cast<uint4*>(op + (size_t)tok * tstride + 8 * cc) = x;
        }
        __syncwarp();
    }
    __device__ __forceinline__ void state_store(const ScanParams& p) const {
        float* dst = p.S_T + sg + (size_t)v * DK + G::SC * part;
#pragma unroll
        for (int c32 = 0; c32 < G::SC / 32; ++c32) {
            float x[32];
            tmem_ld32(tm + lane_base + G::TM_S + G::SC * part + 32 * c32, x);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                reinterpret_cast<float4*>(dst)[8 * c32 + q] =
                    make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
        }
    }
};

// Bounded wait taken by every lane of a warp, with one verdict for the warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, kWaitNs));
}

// Barriers (one block after the record stages), with who arrives and who waits:
//   full[s]  record copy landed      tx count            MMA thread; state warps, before U^T / dec
//   empty[s] stage s read by all     commit              copy thread, before refilling stage s
//            its MMAs (its threads read it before eready)
//   bar1     S [W ; Qg]^T done       commit              state warps, before E^T
//   bar2     E^T Kd accumulated      commit              state warps, before the fp16 copy of S
//   bar3     O^T complete            commit              state warps (outputs)
//   eready   E^T stored, S scaled    one per state warp  MMA thread, before E^T Kd
//   sready   S copy stored           one per state warp  MMA thread, before the next S [W ; Qg]^T
//   drain    error path: completion of every MMA issued so far
// A state warp reads the outputs of chunk m - 2 out of the D1 columns that the first
// product of chunk m overwrites before it arrives on sready for chunk m - 1, which the
// MMA thread waits for before it issues anything of chunk m: that order needs no barrier
// of its own (a separate "outputs read" barrier would also run two phases ahead of the
// MMA thread whenever it lags).  The warp scales S by the decay of chunk m after it has
// read S_m for its fp16 copy (bar2 of chunk m - 1) and before it arrives on eready of
// chunk m, after which E^T Kd of chunk m accumulates onto it.
struct Bars {
    uint64_t *full, *empty, *bar1, *bar2, *bar3, *eready, *sready, *drain;
    uint32_t* tmem_base;
    volatile int* flag;
    volatile int* loaded;   // last chunk whose record copy was issued
    template <int NSTAGE>
    __device__ __forceinline__ static Bars at(uint8_t* p) {
        Bars b;
        b.full = reinterpret_cast<uint64_t*>(p);
        b.empty = b.full + NSTAGE;
        b.bar1 = b.empty + NSTAGE;
        b.bar2 = b.bar1 + 1;
        b.bar3 = b.bar1 + 2;
        b.eready = b.bar1 + 3;
        b.sready = b.bar1 + 4;
        b.drain = b.bar1 + 5;
        b.tmem_base = reinterpret_cast<uint32_t*>(b.bar1 + 6);
        b.flag = reinterpret_cast<volatile int*>(b.bar1 + 7);
        b.loaded = reinterpret_cast<volatile int*>(b.bar1 + 8);
        return b;
    }
};

// One CTA's scan: sequence and head of block index bid.
template <int NW>
__device__ __forceinline__ void scan_cta(const ScanParams& p, int bid) {
    using G = Cfg<NW>;
    constexpr int NSTAGE = G::NSTAGE;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    Tile<NW> t;
    t.sm = sm;
    t.sbase = smem_u32(sm);
    t.h = bid % p.H;
    t.n = bid / p.H;
    const int sp = warp & 3;             // TMEM sub-partition
    t.part = (warp >> 2) % G::NPART;     // key-channel range of the row
    t.v = 32 * sp + lane;                // value row
    t.lane_base = (uint32_t)(32 * sp) << 16;
    t.sg = ((size_t)t.n * p.H + t.h) * DV * DK;
    const Bars b = Bars::at<NSTAGE>(sm + G::OFF_BAR);
    const bool state_thread = warp < NW;
    const bool issuer = tid == 32 * NW;

    long long bos, eos;
    if (!seq_bounds(p.cu_seqlens, t.n, p.T, p.num_seqs, p.dev_status, bos, eos)) return;
    const int nch = (int)((eos - bos + C - 1) / C);

    if (tid == 0) {
        for (int s = 0; s < NSTAGE; ++s) mbar_init(b.full + s, 1), mbar_init(b.empty + s, 1);
        mbar_init(b.bar1, 1);
        mbar_init(b.bar2, 1);
        mbar_init(b.bar3, 1);
        mbar_init(b.eready, NW);
        mbar_init(b.sready, NW);
        mbar_init(b.drain, 1);
        *b.flag = 0;
        *b.loaded = -1;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(b.tmem_base, G::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    t.tm = *b.tmem_base;
    if (state_thread) t.state_init(p);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // everything above overlaps the tail of the WY kernels; records are read below
    pdl_wait();
    const long long first = p.cu_seqlens ? (long long)p.coff[t.n] : (long long)t.n * p.nc;
    int landed = 0;    // issuer: chunks below this one were seen complete on full[]

    if (warp == NW + 1) {
        // ---- the copy thread: stage s takes chunk m once chunk m - NSTAGE's MMAs are done
        if (lane == 0) {
            for (int m = 0; m < nch && m < NSTAGE; ++m) t.load(p, first, m, b.full), *b.loaded = m;
            for (int m = NSTAGE; m < nch && m < NSTAGE + kAhead; ++m) t.prefetch(p, first, m);
            for (int m = NSTAGE; m < nch; ++m) {
                if (*b.flag != 0 ||
                    !mbar_wait(b.empty + m % NSTAGE, (uint32_t)((m / NSTAGE - 1) & 1), kWaitNs)) {
                    *b.flag = 1;
                    break;
                }
                t.load(p, first, m, b.full);
                *b.loaded = m;
                if (m + kAhead < nch) t.prefetch(p, first, m + kAhead);
            }
        }
        __syncwarp();
    } else if (warp == NW) {
        // ---- the MMA thread: waits and issues, nothing else
        if (lane == 0) {
            bool ok = true;
            for (int m = 0; ok && m < nch; ++m) {
                // the fp16 S_m stored (sready of chunk m - 1; it also means the outputs of
                // chunk m - 2 are read out of the D1 columns this chunk overwrites)
                if (m > 0 && !(ok = mbar_wait(b.sready, (uint32_t)((m - 1) & 1), kWaitNs))) break;
                if (!(ok = mbar_wait(b.full + m % NSTAGE, (uint32_t)((m / NSTAGE) & 1), kWaitNs))) break;
                landed = m + 1;
                tc_fence_after();
                t.mma1(m);
                mma_commit(b.bar1);
                if (!(ok = mbar_wait(b.eready, (uint32_t)(m & 1), kWaitNs))) break;
                tc_fence_after();
                t.mma2(m);
                mma_commit(b.bar2);
                t.mma3(m);
                mma_commit(b.bar3);
                mma_commit(b.empty + m % NSTAGE);
            }
            if (!ok) *b.flag = 1;
        }
        __syncwarp();
    } else {
        // ---- state warps: decay of S, E^T, the fp16 copy of S, then the chunk's outputs
        bool ok = true;
        for (int m = 0; m < nch; ++m) {
            if (__any_sync(0xffffffffu, *b.flag != 0)) { ok = false; break; }
            const long long c0 = bos + (long long)m * C;
            const int L = (int)min((long long)C, eos - c0);
            uint4 ut[G::EC / 8];
            if (!(ok = warp_wait(b.full + m % NSTAGE, (uint32_t)((m / NSTAGE) & 1)))) break;
            t.load_ut(m, ut);
            float s_in[G::SC];
            t.decay(m, s_in);
            if (!(ok = warp_wait(b.bar1, (uint32_t)(m & 1)))) break;
            tc_fence_after();
            t.e_step(m, ut);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(b.eready);
            if (p.S_chk) {   // the checkpoint, off the chunk's critical path
                float4* dst = reinterpret_cast<float4*>(p.S_chk + ((size_t)(first + m) * p.H + t.h) * DV * DK +
                                                        (size_t)t.v * DK + G::SC * t.part);
#pragma unroll
                for (int q = 0; q < G::SC / 4; ++q)
                    dst[q] = make_float4(s_in[4 * q], s_in[4 * q + 1], s_in[4 * q + 2], s_in[4 * q + 3]);
            }
            if (!(ok = warp_wait(b.bar2, (uint32_t)(m & 1)))) break;
            tc_fence_after();
            t.s_copy();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(b.sready);
            if (!(ok = warp_wait(b.bar3, (uint32_t)(m & 1)))) break;
            tc_fence_after();
            t.read_out(p, m, c0, L, warp);
            tc_fence_before();
        }
        if (!ok && lane == 0) *b.flag = 1;
    }
    tc_fence_before();
    __syncthreads();
    if (*b.flag != 0) {
        if (p.dev_status && tid == 0) atomicOr(p.dev_status, KDA_DEV_TIMEOUT);
        // let copies / MMAs still in flight land before the memory goes away
        if (issuer) {
            mma_commit(b.drain);
            (void)mbar_wait(b.drain, 0, kWaitNs);
            const int loaded = *b.loaded;
            for (int c = landed; c <= loaded; ++c)
                (void)mbar_wait(b.full + c % NSTAGE, (uint32_t)((c / NSTAGE) & 1), kWaitNs);
        }
    } else if (state_thread && p.S_T) {
        tc_fence_after();
        t.state_store(p);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(t.tm, G::TMEM_COLS);
    }
}

}  // namespace
}  // namespace kda
