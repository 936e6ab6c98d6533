// kda_chunk_bwd_scan.cu -- the sequential half of the chunkwise backward: the
// reverse state-gradient scan.
//
// The chunk map of the forward (kda_chunk_record.cuh) is
//
//   E = U - W S^T,   O = Qg S^T + Aqk E,   S' = S Diag(dec) + E^T Kd,
//
// so for the loss sum(out * dO) + sum(S_T * dS_T), with dS' the gradient of a
// chunk's outgoing state, the gradient of its incoming state follows from the
// same record operands (the pages give no backward derivation; this is the chain
// rule of the chunk map, checked in float64 against autograd of the token loop):
//
//   dE^T = dS' Kd^T + dO^T Aqk                      (d_v x C)
//   dS   = dS' Diag(dec) + dO^T Qg - dE^T W         (d_v x d_k)
//
// One CTA per (sequence, head) walks the chunks from last to first, with dS held
// the way the forward scan holds S: one value row per tensor-memory lane, the
// fp32 dS the accumulator of its own update and its fp16 copy the A operand of
// the next (earlier) chunk's first product, as are dO^T and dE^T.  For every chunk
// it leaves dS' (the gradient of the chunk's outgoing state) and dE in the
// workspace for the chunk-parallel gradient kernels, and writes dS0 at the end.
// dE^T enters the dS update negated (its fp16 copy is stored as -dE^T), so every
// product accumulates.
//
// Roles and barriers mirror kda_chunk_scan.cu: 16 state warps, one MMA thread,
// one copy thread; each barrier completes once per chunk step.
#include "kda_chunk_bwd.cuh"
#include "kda_chunk_record.cuh"
#include "kda_chunk_scan.cuh"
#include "kda_internal.cuh"
#include "kda_tc_common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {
namespace rv {   // the reverse scan (the forward scan's device code comes from kda_chunk_scan.cuh)

using namespace sm100;
using namespace tc;

constexpr int C = rec::C, DK = rec::DK, DV = rec::DV;
constexpr uint64_t kWaitNs = 1000000000ull;   // 1 s bound on every wait
constexpr int NW = 16;                         // state warps: 4 sub-partitions x 4 channel ranges
constexpr int NPART = NW / 4, SC = DK / NPART, EC = C / NPART;
constexpr int NT = 32 * NW + 64;               // + the MMA warp + the copy warp
constexpr int NSTAGE = 2;
constexpr int REC_STAGE = (rec::BYTES + 1023) / 1024 * 1024;
constexpr int DO_BYTES = C * DV * 2;           // the chunk's dO tile, bf16 [token][v]
constexpr int STAGE = REC_STAGE + DO_BYTES;
constexpr int OFF_BAR = NSTAGE * STAGE;
constexpr int SMEM_BYTES = OFF_BAR + 128 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory over the sm_100 per-block limit");
constexpr uint32_t TM_DS = 0;      // 128 cols: fp32 dS (accumulator of its update)
constexpr uint32_t TM_DE = 128;    // 64 cols: dE^T
constexpr uint32_t TM_AS = 192;    // 64 cols: fp16 dS' (A operand, K = key channel)
constexpr uint32_t TM_AE = 256;    // 32 cols: fp16 dE^T (A operand, K = token)
constexpr uint32_t TM_AO = 288;    // 32 cols: fp16 dO^T (A operand, K = token)
constexpr uint32_t TMEM_COLS = 512;

struct BwdScanParams {
    CUtensorMap map_do;
    const uint8_t* rec;
    const int32_t* coff;
    const int32_t* cu_seqlens;
    const float* d_ST;
    float* dS0;
    float* dsp;      // [slot][H][d_v][d_k] fp32: gradient of each chunk's outgoing state
    float* de;       // [slot][H][C][d_v] fp32: dE of each chunk
    int32_t* dev_status;
    int T, H, num_seqs, nc;
};

struct Bars {
    uint64_t *full, *empty, *oready, *bar1, *eready, *bar2, *sready, *drain;
    uint32_t* tmem_base;
    volatile int* flag;
    volatile int* loaded;
    __device__ __forceinline__ static Bars at(uint8_t* p) {
        Bars b;
        b.full = reinterpret_cast<uint64_t*>(p);
        b.empty = b.full + NSTAGE;
        b.oready = b.empty + NSTAGE;
        b.bar1 = b.oready + 1;
        b.eready = b.bar1 + 1;
        b.bar2 = b.eready + 1;
        b.sready = b.bar2 + 1;
        b.drain = b.sready + 1;
        b.tmem_base = reinterpret_cast<uint32_t*>(b.drain + 1);
        b.flag = reinterpret_cast<volatile int*>(b.drain + 2);
        b.loaded = reinterpret_cast<volatile int*>(b.drain + 3);
        return b;
    }
};
static_assert(8 * (2 * NSTAGE + 9) <= 128, "barrier block");

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, kWaitNs));
}

// Barriers, step r = 0, 1, ... walks chunk m = nch - 1 - r:
//   full[s]  record + dO tile landed   tx count            MMA thread; state warps
//   empty[s] stage s read by its MMAs  commit              copy thread, before refilling stage s
//   oready   dO^T stored, dS scaled    one per state warp  MMA thread, before dE^T
//   bar1     dE^T done                 commit              state warps
//   eready   fp16 dE^T stored          one per state warp  MMA thread, before the dS update
//   bar2     dS update done            commit              state warps
//   sready   fp16 dS stored            one per state warp  MMA thread, before the next step's dE^T
// The state warps read a stage (dO tile, dec) before oready, and everything they
// write to tensor memory in step r is read by MMAs of step r that complete before
// the warps' next write (bar1 / bar2 of step r precede it in their program order).
// One CTA's reverse scan: sequence and head of block index bid.
__device__ __forceinline__ void bwd_scan_cta(const BwdScanParams& p, int bid) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = bid % p.H, n = bid / p.H;
    const int sp = warp & 3, part = (warp >> 2) % NPART;
    const int v = 32 * sp + lane;
    const uint32_t lane_base = (uint32_t)(32 * sp) << 16;
    const uint32_t sbase = smem_u32(sm);
    const size_t sg = ((size_t)n * p.H + h) * DV * DK;
    const Bars b = Bars::at(sm + OFF_BAR);

    long long bos, eos;
    if (!seq_bounds(p.cu_seqlens, n, p.T, p.num_seqs, p.dev_status, bos, eos)) return;
    const int nch = (int)((eos - bos + C - 1) / C);

    if (tid == 0) {
        for (int s = 0; s < NSTAGE; ++s) mbar_init(b.full + s, 1), mbar_init(b.empty + s, 1);
        mbar_init(b.oready, NW);
        mbar_init(b.bar1, 1);
        mbar_init(b.eready, NW);
        mbar_init(b.bar2, 1);
        mbar_init(b.sready, NW);
        mbar_init(b.drain, 1);
        *b.flag = 0;
        *b.loaded = -1;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(b.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *b.tmem_base;
    pdl_wait();   // d_ST, the records and the checkpoints are complete from here on
    if (warp < NW) {
        // dS = dS_T (or zero) and its fp16 copy
        const float* src = p.d_ST ? p.d_ST + sg + (size_t)v * DK + SC * part : nullptr;
        uint32_t x[32], r[16];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 f = src ? reinterpret_cast<const float4*>(src)[q] : make_float4(0.f, 0.f, 0.f, 0.f);
            x[4 * q] = __float_as_uint(f.x); x[4 * q + 1] = __float_as_uint(f.y);
            x[4 * q + 2] = __float_as_uint(f.z); x[4 * q + 3] = __float_as_uint(f.w);
            r[2 * q] = pack_f16(f.x, f.y);
            r[2 * q + 1] = pack_f16(f.z, f.w);
        }
        tmem_st32(tm + lane_base + TM_DS + SC * part, x);
        tmem_st16(tm + lane_base + TM_AS + (SC / 2) * part, r);
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const long long first = p.cu_seqlens ? (long long)p.coff[n] : (long long)n * p.nc;
    auto chunk_of = [&](int r) { return nch - 1 - r; };
    auto stage_of = [&](int r) { return sm + (r % NSTAGE) * STAGE; };
    int landed = 0;

    if (warp == NW + 1) {
        // ---- the copy thread: record and dO tile of step r into stage r % NSTAGE
        if (lane == 0) {
            auto load = [&](int r) {
                const int m = chunk_of(r);
                uint64_t* bar = b.full + (r % NSTAGE);
                uint8_t* st = stage_of(r);
                mbar_arrive_expect_tx(bar, (uint32_t)(rec::BYTES + DO_BYTES));
                bulk_load(st, p.rec + ((size_t)(first + m) * p.H + h) * rec::BYTES, (uint32_t)rec::BYTES, bar);
                tma_load_3d(st + REC_STAGE, &p.map_do, bar, 0, h, (int)(bos + (long long)m * C));
                *b.loaded = r;
            };
            for (int r = 0; r < nch && r < NSTAGE; ++r) load(r);
            for (int r = NSTAGE; r < nch; ++r) {
                if (*b.flag != 0 || !mbar_wait(b.empty + r % NSTAGE, (uint32_t)((r / NSTAGE - 1) & 1), kWaitNs)) {
                    *b.flag = 1;
                    break;
                }
                load(r);
            }
        }
        __syncwarp();
    } else if (warp == NW) {
        // ---- the MMA thread
        if (lane == 0) {
            bool ok = true;
            for (int r = 0; ok && r < nch; ++r) {
                if (r > 0 && !(ok = mbar_wait(b.sready, (uint32_t)((r - 1) & 1), kWaitNs))) break;
                if (!(ok = mbar_wait(b.full + r % NSTAGE, (uint32_t)((r / NSTAGE) & 1), kWaitNs))) break;
                landed = r + 1;
                if (!(ok = mbar_wait(b.oready, (uint32_t)(r & 1), kWaitNs))) break;
                tc_fence_after();
                const uint32_t st = sbase + (uint32_t)((r % NSTAGE) * STAGE);
                // dE^T = dS' Kd^T (Kd rows are tokens j, K-major over the channel) + dO^T Aqk
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_tmem_a(tm + TM_DE, tm + TM_AS + 8u * s, rowview_desc(st + rec::KD, s),
                               idesc_f16(128, 64, false, false), s > 0);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_tmem_a(tm + TM_DE, tm + TM_AO + 8u * s, mnmaj_desc(st + rec::AQ, 64, s),
                               idesc_f16(128, 64, false, true), 1);
                mma_commit(b.bar1);
                if (!(ok = mbar_wait(b.eready, (uint32_t)(r & 1), kWaitNs))) break;
                tc_fence_after();
                // dS += dO^T Qg + (-dE^T) W (Qg, W rows are tokens: MN-major over the channel)
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_tmem_a(tm + TM_DS, tm + TM_AO + 8u * s, mnmaj_desc(st + rec::WQ + 16384, 128, s),
                               idesc_f16(128, 128, false, true), 1);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_tmem_a(tm + TM_DS, tm + TM_AE + 8u * s, mnmaj_desc(st + rec::WQ, 128, s),
                               idesc_f16(128, 128, false, true), 1);
                mma_commit(b.bar2);
                mma_commit(b.empty + r % NSTAGE);
            }
            if (!ok) *b.flag = 1;
        }
        __syncwarp();
    } else {
        // ---- state warps
        bool ok = true;
        for (int r = 0; r < nch; ++r) {
            if (__any_sync(0xffffffffu, *b.flag != 0)) { ok = false; break; }
            const int m = chunk_of(r);
            const long long c0 = bos + (long long)m * C;
            const int L = (int)min((long long)C, eos - c0);
            const size_t slot_h = (size_t)(first + m) * p.H + h;
            if (!(ok = warp_wait(b.full + r % NSTAGE, (uint32_t)((r / NSTAGE) & 1)))) break;
            const uint8_t* st = stage_of(r);
            // the global writes of dS' and dE come after the arrive that releases the
            // MMA thread: they leave the chunk's critical path
            float x[32];
            {
                // dO^T of this thread's tokens (rows past the chunk's length are zero)
                const __nv_bfloat16* dot = reinterpret_cast<const __nv_bfloat16*>(st + REC_STAGE);
                uint32_t o[EC / 2];
#pragma unroll
                for (int e = 0; e < EC / 2; ++e) {
                    const int i = EC * part + 2 * e;
                    const float a = i < L ? __bfloat162float(dot[i * DV + v]) : 0.f;
                    const float c = i + 1 < L ? __bfloat162float(dot[(i + 1) * DV + v]) : 0.f;
                    o[e] = pack_f16(a, c);
                }
                tmem_st8(tm + lane_base + TM_AO + (EC / 2) * part, o);
                // dS' Diag(dec)
                const float4* dec = reinterpret_cast<const float4*>(st + rec::DEC) + (SC / 4) * part;
                tmem_ld32(tm + lane_base + TM_DS + SC * part, x);
                uint32_t y[32];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 g = dec[q];
                    y[4 * q] = __float_as_uint(x[4 * q] * g.x);
                    y[4 * q + 1] = __float_as_uint(x[4 * q + 1] * g.y);
                    y[4 * q + 2] = __float_as_uint(x[4 * q + 2] * g.z);
                    y[4 * q + 3] = __float_as_uint(x[4 * q + 3] * g.w);
                }
                tmem_st32(tm + lane_base + TM_DS + SC * part, y);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(b.oready);
            {
                float4* out = reinterpret_cast<float4*>(p.dsp + slot_h * DV * DK + (size_t)v * DK + SC * part);
#pragma unroll
                for (int q = 0; q < 8; ++q) out[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
            }
            if (!(ok = warp_wait(b.bar1, (uint32_t)(r & 1)))) break;
            tc_fence_after();
            float d[EC];
            {
                // fp16 -dE^T of this thread's tokens
                tmem_ld16(tm + lane_base + TM_DE + EC * part, d);
                uint32_t r16[EC / 2];
#pragma unroll
                for (int e = 0; e < EC / 2; ++e) r16[e] = pack_f16(-d[2 * e], -d[2 * e + 1]);
                tmem_st8(tm + lane_base + TM_AE + (EC / 2) * part, r16);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(b.eready);
            {
                // dE to the workspace, token-major: one coalesced row of the warp's 32
                // values per token
                float* de = p.de + (slot_h * C + EC * part) * DV + v;
#pragma unroll
                for (int e = 0; e < EC; ++e) de[(size_t)e * DV] = d[e];
            }
            if (!(ok = warp_wait(b.bar2, (uint32_t)(r & 1)))) break;
            tc_fence_after();
            {
                float x[32];
                tmem_ld32(tm + lane_base + TM_DS + SC * part, x);
                uint32_t r16[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) r16[i] = pack_f16(x[2 * i], x[2 * i + 1]);
                tmem_st16(tm + lane_base + TM_AS + (SC / 2) * part, r16);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(b.sready);
        }
        if (!ok && lane == 0) *b.flag = 1;
    }
    tc_fence_before();
    __syncthreads();
    if (*b.flag != 0) {
        if (p.dev_status && tid == 0) atomicOr(p.dev_status, KDA_DEV_TIMEOUT);
        if (tid == 32 * NW) {
            mma_commit(b.drain);
            (void)mbar_wait(b.drain, 0, kWaitNs);
            const int loaded = *b.loaded;
            for (int r = landed; r <= loaded; ++r)
                (void)mbar_wait(b.full + r % NSTAGE, (uint32_t)((r / NSTAGE) & 1), kWaitNs);
        }
    } else if (warp < NW && p.dS0) {
        tc_fence_after();
        float x[32];
        tmem_ld32(tm + lane_base + TM_DS + SC * part, x);
        float4* dst = reinterpret_cast<float4*>(p.dS0 + sg + (size_t)v * DK + SC * part);
#pragma unroll
        for (int q = 0; q < 8; ++q) dst[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, TMEM_COLS);
    }
}

}  // namespace rv

// The backward's two scans in one launch: CTAs [0, fwd_ctas) run the forward scan
// (checkpoints, no outputs), the rest the reverse scan.  The reverse scan needs only
// the records, dO and d_ST, so the two are independent and share the GPU, each
// having one CTA per (sequence, head).
struct DualScanParams {
    ScanParams f;
    rv::BwdScanParams b;
    int fwd_ctas;
};
static_assert(Cfg<16>::NT == rv::NT, "the two scans run the same block shape");
constexpr int kDualSmem = Cfg<16>::SMEM_BYTES > rv::SMEM_BYTES ? Cfg<16>::SMEM_BYTES : rv::SMEM_BYTES;

__global__ void __launch_bounds__(rv::NT, 1) kda_chunk_fwdbwd_scan_kernel(const __grid_constant__ DualScanParams p) {
    if ((int)blockIdx.x < p.fwd_ctas) {
        scan_cta<16>(p.f, (int)blockIdx.x);
    } else {
        rv::bwd_scan_cta(p.b, (int)blockIdx.x - p.fwd_ctas);
    }
}

}  // namespace

cudaError_t launch_chunk_scans_bwd(const ChunkBwdArgs& a, const uint8_t* ws, const BwdLayout& bl, cudaStream_t st) {
    using rv::BwdScanParams;
    using rv::NT;
    const rec::Layout& lay = bl.fwd;
    DualScanParams d;
    memset(&d, 0, sizeof(d));
    ScanParams& f = d.f;
    f.rec = ws + lay.rec_off;
    f.coff = a.cu_seqlens ? reinterpret_cast<const int32_t*>(ws + lay.coff_off) : nullptr;
    f.cu_seqlens = a.cu_seqlens;
    f.S0 = a.S0;
    f.S_T = nullptr;
    f.out = nullptr;
    f.S_chk = reinterpret_cast<float*>(const_cast<uint8_t*>(ws) + bl.chk_off);
    f.dev_status = a.dev_status;
    f.T = a.T;
    f.H = a.H;
    f.num_seqs = a.num_seqs;
    f.nc = (a.T + rec::C - 1) / rec::C;
    BwdScanParams& p = d.b;
    p.rec = ws + lay.rec_off;
    p.coff = f.coff;
    p.cu_seqlens = a.cu_seqlens;
    p.d_ST = a.d_ST;
    p.dS0 = a.dS0;
    p.dsp = reinterpret_cast<float*>(const_cast<uint8_t*>(ws) + bl.dsp_off);
    p.de = reinterpret_cast<float*>(const_cast<uint8_t*>(ws) + bl.de_off);
    p.dev_status = a.dev_status;
    p.T = a.T;
    p.H = a.H;
    p.num_seqs = a.num_seqs;
    p.nc = f.nc;
    const long long tokens = (long long)a.B * a.T;
    if (tokens > 0 && !make_map(&p.map_do, a.d_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rec::DV, a.H, tokens, rec::DV, rec::C,
                                CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const long long pairs = (long long)a.num_seqs * a.H;
    d.fwd_ctas = (int)pairs;
    cudaError_t e = cudaFuncSetAttribute(kda_chunk_fwdbwd_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kDualSmem);
    if (e != cudaSuccess) return e;
    return launch_after(kda_chunk_fwdbwd_scan_kernel, dim3((unsigned)(2 * pairs)), NT, kDualSmem, st, d);
}

}  // namespace kda
