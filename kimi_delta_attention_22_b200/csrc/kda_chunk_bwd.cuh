// kda_chunk_bwd.cuh -- launch interfaces and workspace layout of the chunkwise
// backward (gradients of the tensor-core prefill; d_k = d_v = 128, chunk 64).
//
// The backward runs four kernels (five launches) on one stream:
//   1. the forward's WY kernel, both launches: every chunk's record (kda_chunk_record.cuh);
//   2. one launch of two independent scans side by side (kda_chunk_bwd_scan.cu): the
//      forward's state scan with outputs off, keeping every chunk's incoming state
//      S_c (fp32) in the workspace, and the reverse state scan: dS0, and per chunk
//      the gradient of its outgoing state dS' and dE;
//   3. and 4. the chunk-parallel gradient kernels (kda_chunk_bwd_grad.cu): per
//      (chunk, head), the triangular-solve half (E, the solve's gradient, dv,
//      dbeta) and then the rest (dq, dk, dg); their products run on the tensor
//      cores, the decay-weighted Gram parts too where one decay reference holds
//      the chunk (on CUDA cores in fp32 otherwise).
#pragma once

#include "kda_chunk_record.cuh"
#include "kda_internal.cuh"

namespace kda {

struct ChunkBwdArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    const float* S0;
    const int32_t* cu_seqlens;
    const void* d_out;
    const float* d_ST;    // may be null (zero)
    float* dq;            // [tok][Hk][d_k]
    float* dk;
    float* dv;            // [tok][H][d_v]
    float* dg;            // the shape of g; null without a gate
    float* dbeta;         // [tok][H]
    float* dS0;           // may be null
    int32_t* dev_status;
    int B, T, H, Hk, num_seqs, gate;
    float scale;
};

// Workspace: the forward's records (rec::layout), then per (slot, head):
//   chk  fp32 [d_v][d_k]  incoming state of the chunk
//   dsp  fp32 [d_v][d_k]  gradient of the chunk's outgoing state
//   de   fp32 [C][d_v]    dE from the reverse scan
//   e16  2 x 16 KB        E as a two-term fp16 expansion (hi, then lo = E - hi), each the
//                         byte image of a K-major 64 x 128 MMA operand tile
//   pr16 16 KB            dPr = -diag(beta) dEbar, one such image (fp16)
//   da   fp32 [C][C]      dA = diag(beta) dL (strictly lower)
struct BwdLayout {
    rec::Layout fwd;
    size_t chk_off, dsp_off, de_off, e16_off, pr16_off, da_off, bytes;
};

constexpr size_t kTile16 = (size_t)rec::C * rec::DV * 2;   // one fp16 64 x 128 operand image

inline BwdLayout bwd_layout(int B, int T, int H, int num_seqs, bool varlen) {
    BwdLayout b;
    b.fwd = rec::layout(B, T, H, num_seqs, varlen);
    const size_t units = (size_t)b.fwd.slots * H;
    const size_t st = (size_t)rec::DV * rec::DK * sizeof(float);
    const size_t vc = (size_t)rec::DV * rec::C * sizeof(float);
    const size_t cc = (size_t)rec::C * rec::C * sizeof(float);
    b.chk_off = rec::round256(b.fwd.bytes);
    b.dsp_off = b.chk_off + units * st;
    b.de_off = b.dsp_off + units * st;
    b.e16_off = b.de_off + units * vc;
    b.pr16_off = b.e16_off + units * 2 * kTile16;
    b.da_off = b.pr16_off + units * kTile16;
    b.bytes = b.da_off + units * cc;
    return b;
}

inline ChunkArgs forward_args(const ChunkBwdArgs& a) {
    ChunkArgs f = {};
    f.q = a.q;
    f.k = a.k;
    f.v = a.v;
    f.g = a.g;
    f.beta = a.beta;
    f.S0 = a.S0;
    f.cu_seqlens = a.cu_seqlens;
    f.out = nullptr;
    f.S_T = nullptr;
    f.dev_status = a.dev_status;
    f.B = a.B;
    f.T = a.T;
    f.H = a.H;
    f.d_k = rec::DK;
    f.d_v = rec::DV;
    f.num_seqs = a.num_seqs;
    f.gate = a.gate;
    f.chunk = rec::C;
    f.Hk = a.Hk;
    f.scale = a.scale;
    return f;
}

// The forward scan with checkpoints (no outputs) and the reverse scan, in one launch.
cudaError_t launch_chunk_scans_bwd(const ChunkBwdArgs& a, const uint8_t* ws, const BwdLayout& bl, cudaStream_t st);
cudaError_t launch_chunk_bwd_grad(const ChunkBwdArgs& a, uint8_t* ws, const BwdLayout& bl, cudaStream_t st);

}  // namespace kda
