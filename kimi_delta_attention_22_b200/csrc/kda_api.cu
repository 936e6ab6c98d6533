// kda_api.cu -- the C ABI of include/kda.h: host-side validation and kernel
// selection.  Every check runs before any launch, so a rejected call launches
// nothing, and nothing here synchronises.  The only memory this file obtains is
// the tensor-core prefill's scratch when the caller passes no workspace: it is
// taken from the device's stream-ordered pool (cudaMallocAsync) and given back
// on the same stream after the kernels that use it.
#include <atomic>
#include <stdint.h>

#include "kda_chunk_bwd.cuh"
#include "kda_internal.cuh"

namespace kda {
size_t chunk_f32_smem_bytes(int C, int D, int V);
}  // namespace kda

namespace {

// Scratch of kda_chunk_fwd_noalloc: a file-scope device array that every device
// which loads this module holds until the process exits.  160 MiB holds the records
// of 2,200+ (chunk, head) pairs (e.g. 4 sequences x 16 heads x 2048 tokens).
constexpr size_t kStaticScratchBytes = (size_t)160 << 20;
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];
// Its device address, resolved once per device (host code cannot use the symbol itself).
constexpr int kMaxDevices = 64;
std::atomic<void*> g_static_scratch_addr[kMaxDevices];

// The tensor-core prefill: bf16 q/k/v with d_k = d_v = 128 and chunks of 64.
bool tc_supports(int D, int V, int C) { return D == 128 && V == 128 && C == 64; }

bool aligned16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool f32path_supports(int D, int V, int C) {
    return D >= 16 && D <= 128 && D % 16 == 0 && V >= 16 && V <= 128 && V % 16 == 0 &&
           (C == 16 || C == 32 || C == 64);
}

kda_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

// Query/key heads of a shape (0 means one per value head); -1 if they do not divide H.
int qk_heads_of(const kda_shape_t* sh) {
    const int Hk = sh->qk_heads == 0 ? sh->H : sh->qk_heads;
    return (Hk > 0 && sh->H > 0 && sh->H % Hk == 0) ? Hk : -1;
}

}  // namespace

extern "C" {

const char* kda_status_str(kda_status_t s) {
    switch (s) {
        case KDA_OK: return "ok";
        case KDA_ERR_INVALID_ARG: return "invalid argument";
        case KDA_ERR_UNSUPPORTED: return "unsupported shape, chunk or dtype";
        case KDA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case KDA_ERR_CUDA: return "CUDA launch error";
        case KDA_ERR_TIMEOUT: return "bounded device wait expired";
        case KDA_ERR_TOO_LARGE: return "shape needs more scratch than the library's static array holds";
    }
    return "unknown status";
}

const char* kda_version(void) { return "libkda 0.2 (sm_100a)"; }

size_t kda_chunk_fwd_workspace_size(const kda_shape_t* sh, int varlen) {
    if (sh == nullptr || sh->B < 0 || sh->T < 0 || sh->H <= 0 || sh->num_seqs < 0) return 0;
    if (sh->dtype != KDA_BF16 || !tc_supports(sh->d_k, sh->d_v, sh->chunk)) return 0;
    return kda::rec::layout(sh->B, sh->T, sh->H, sh->num_seqs, varlen != 0).bytes;
}

kda_status_t kda_chunk_fwd(const kda_shape_t* sh, const void* q, const void* k, const void* v,
                           const float* g, const float* beta, const float* S0,
                           const int32_t* cu_seqlens, void* out, float* S_T, void* workspace,
                           size_t workspace_bytes, void* stream) {
    if (sh == nullptr) return KDA_ERR_INVALID_ARG;
    const int B = sh->B, T = sh->T, H = sh->H, D = sh->d_k, V = sh->d_v, N = sh->num_seqs;
    if (B < 0 || T < 0 || H <= 0 || D <= 0 || V <= 0 || N < 0) return KDA_ERR_INVALID_ARG;
    const int Hk = qk_heads_of(sh);
    if (Hk < 0) return KDA_ERR_INVALID_ARG;
    if (sh->dtype != KDA_F32 && sh->dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (sh->gate != KDA_GATE_CHANNEL && sh->gate != KDA_GATE_SCALAR && sh->gate != KDA_GATE_NONE)
        return KDA_ERR_INVALID_ARG;
    if ((sh->gate == KDA_GATE_NONE) != (g == nullptr)) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens == nullptr) {
        if (N != B) return KDA_ERR_INVALID_ARG;
    } else if (B != 1) {
        return KDA_ERR_INVALID_ARG;
    }
    if ((long long)B * T > 0 && (!q || !k || !v || !beta || !out)) return KDA_ERR_INVALID_ARG;
    const bool g_vec = sh->gate == KDA_GATE_CHANNEL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !(g_vec ? aligned16(g) : aligned4(g)) ||
        !aligned4(beta) || !aligned16(S0) || !aligned4(cu_seqlens) || !aligned16(out) ||
        !aligned16(S_T))
        return KDA_ERR_MISALIGNED;
    if ((long long)N * H * 2 > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;

    const bool bf16 = sh->dtype == KDA_BF16;
    const int C = sh->chunk;
    const bool tc = bf16 && tc_supports(D, V, C);
    if (!tc && !f32path_supports(D, V, C)) return KDA_ERR_UNSUPPORTED;
    kda::rec::Layout lay{};
    if (tc) {
        lay = kda::rec::layout(B, T, H, N, cu_seqlens != nullptr);
        if (lay.slots * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
        if (workspace != nullptr) {
            if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_MISALIGNED;
            if (workspace_bytes < lay.bytes) return KDA_ERR_INVALID_ARG;
        }
    }
    if (N == 0) return KDA_OK;

    kda::ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S0 = S0; a.cu_seqlens = cu_seqlens;
    a.out = out; a.S_T = S_T; a.dev_status = sh->dev_status;
    a.B = B; a.T = T; a.H = H; a.d_k = D; a.d_v = V; a.num_seqs = N; a.gate = sh->gate;
    a.chunk = C;
    a.Hk = Hk;
    a.scale = 1.0f / sqrtf((float)D);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!tc) return from_cuda(kda::launch_chunk_f32path(a, bf16, st));
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const bool pooled = ws == nullptr;   // scratch from the stream-ordered pool (256-byte aligned)
    if (pooled && cudaMallocAsync(reinterpret_cast<void**>(&ws), lay.bytes, st) != cudaSuccess)
        return KDA_ERR_CUDA;
    cudaError_t e = kda::launch_chunk_wy(a, ws, lay, st);
    if (e == cudaSuccess) e = kda::launch_chunk_scan(a, ws, lay, st);
    if (pooled) {
        const cudaError_t f = cudaFreeAsync(ws, st);
        if (e == cudaSuccess) e = f;
    }
    return from_cuda(e);
}

kda_status_t kda_chunk_fwd_noalloc(const kda_shape_t* sh, const void* q, const void* k,
                                   const void* v, const float* g, const float* beta, const float* S0,
                                   const int32_t* cu_seqlens, void* out, float* S_T, void* stream) {
    if (sh == nullptr) return KDA_ERR_INVALID_ARG;
    const size_t need = kda_chunk_fwd_workspace_size(sh, cu_seqlens != nullptr);
    // Shapes without scratch (the CUDA-core path), empty batches and invalid shapes go
    // straight through: kda_chunk_fwd validates them and, for them, takes no memory.
    if (need == 0 || sh->num_seqs <= 0)
        return kda_chunk_fwd(sh, q, k, v, g, beta, S0, cu_seqlens, out, S_T, nullptr, 0, stream);
    if (need > kStaticScratchBytes) return KDA_ERR_TOO_LARGE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
    void* ws = g_static_scratch_addr[dev].load(std::memory_order_acquire);
    if (ws == nullptr) {
        // set-up on this device's first call: the array's device address (loading the
        // module and with it the array, if nothing on this device has yet)
        if (cudaGetSymbolAddress(&ws, g_static_scratch) != cudaSuccess || ws == nullptr) return KDA_ERR_CUDA;
        g_static_scratch_addr[dev].store(ws, std::memory_order_release);
    }
    return kda_chunk_fwd(sh, q, k, v, g, beta, S0, cu_seqlens, out, S_T, ws, kStaticScratchBytes, stream);
}

kda_status_t kda_recurrent_fwd(const kda_shape_t* sh, const void* q, const void* k, const void* v,
                               const float* g, const float* beta, float* S, void* out, void* stream) {
    if (sh == nullptr) return KDA_ERR_INVALID_ARG;
    const int N = sh->B, T = sh->T, H = sh->H, D = sh->d_k, V = sh->d_v;
    if (N < 0 || T < 0 || H <= 0 || D <= 0 || V <= 0 || sh->num_seqs != N) return KDA_ERR_INVALID_ARG;
    const int Hk = qk_heads_of(sh);
    if (Hk < 0) return KDA_ERR_INVALID_ARG;
    if (sh->dtype != KDA_F32 && sh->dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (sh->gate != KDA_GATE_CHANNEL && sh->gate != KDA_GATE_SCALAR && sh->gate != KDA_GATE_NONE)
        return KDA_ERR_INVALID_ARG;
    if ((sh->gate == KDA_GATE_NONE) != (g == nullptr)) return KDA_ERR_INVALID_ARG;
    if (N > 0 && (!S || (T > 0 && (!q || !k || !v || !beta || !out)))) return KDA_ERR_INVALID_ARG;
    const bool g_vec = sh->gate == KDA_GATE_CHANNEL;
    if (!aligned16(q) || !aligned16(k) || !aligned4(v) || !(g_vec ? aligned16(g) : aligned4(g)) ||
        !aligned4(beta) || !aligned16(S) || !aligned4(out))
        return KDA_ERR_MISALIGNED;
    if (D != 128 || V > 65535 * 128) return KDA_ERR_UNSUPPORTED;
    if ((long long)N * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    if (N == 0 || T == 0) return KDA_OK;
    if (T == 1) {
        // one token per sequence: [N, 1, H, .] is the decode step's [N, H, .] layout, and its
        // kernel streams the state at the copy rate (the two are the same arithmetic)
        kda::DecodeArgs d;
        d.q = q; d.k = k; d.v = v; d.g = g; d.beta = beta; d.S = S; d.out = out;
        d.N = N; d.H = H; d.d_k = D; d.d_v = V; d.gate = sh->gate;
        d.Hk = Hk;
        d.scale = 1.0f / sqrtf((float)D);
        return from_cuda(kda::launch_decode(d, sh->dtype == KDA_BF16, static_cast<cudaStream_t>(stream)));
    }

    kda::RecurrentArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S = S; a.out = out;
    a.N = N; a.T = T; a.H = H; a.d_k = D; a.d_v = V; a.gate = sh->gate;
    a.Hk = Hk;
    a.scale = 1.0f / sqrtf((float)D);
    return from_cuda(kda::launch_recurrent(a, sh->dtype == KDA_BF16, static_cast<cudaStream_t>(stream)));
}

size_t kda_recurrent_bwd_workspace_size(const kda_shape_t* sh) {
    if (sh == nullptr || sh->B <= 0 || sh->T <= 0 || sh->H <= 0 || sh->d_v <= 0) return 0;
    return kda::recurrent_bwd_workspace_bytes(sh->B, sh->T, sh->H, sh->d_v);
}

kda_status_t kda_recurrent_bwd(const kda_shape_t* sh, const void* q, const void* k, const void* v,
                               const float* g, const float* beta, const float* S0, const void* d_out,
                               const float* d_ST, float* dq, float* dk, float* dv, float* dg,
                               float* dbeta, float* dS0, void* workspace, size_t workspace_bytes,
                               void* stream) {
    if (sh == nullptr) return KDA_ERR_INVALID_ARG;
    const int N = sh->B, T = sh->T, H = sh->H, D = sh->d_k, V = sh->d_v;
    if (N < 0 || T < 0 || H <= 0 || D <= 0 || V <= 0 || sh->num_seqs != N) return KDA_ERR_INVALID_ARG;
    const int Hk = qk_heads_of(sh);
    if (Hk < 0) return KDA_ERR_INVALID_ARG;
    if (sh->dtype != KDA_F32 && sh->dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (sh->gate != KDA_GATE_CHANNEL && sh->gate != KDA_GATE_SCALAR && sh->gate != KDA_GATE_NONE)
        return KDA_ERR_INVALID_ARG;
    const bool gated = sh->gate != KDA_GATE_NONE;
    if (gated != (g != nullptr) || gated != (dg != nullptr)) return KDA_ERR_INVALID_ARG;
    const bool any = (long long)N * T > 0;
    if (any && (!q || !k || !v || !beta || !d_out || !dq || !dk || !dv || !dbeta)) return KDA_ERR_INVALID_ARG;
    if (!aligned4(q) || !aligned4(k) || !aligned4(v) || !aligned4(g) || !aligned4(beta) || !aligned4(d_out) ||
        !aligned16(S0) || !aligned16(d_ST) || !aligned4(dq) || !aligned4(dk) || !aligned4(dv) ||
        !aligned4(dg) || !aligned4(dbeta) || !aligned16(dS0) || !aligned16(workspace))
        return KDA_ERR_MISALIGNED;
    if (D != 128 || V > 65535 * 16) return KDA_ERR_UNSUPPORTED;
    if ((long long)N * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    if (N == 0) return KDA_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {   // no tokens: S_T = S0, so dS0 = d_ST
        if (!dS0) return KDA_OK;
        const size_t nb = (size_t)N * H * V * D * sizeof(float);
        return from_cuda(d_ST ? cudaMemcpyAsync(dS0, d_ST, nb, cudaMemcpyDeviceToDevice, st)
                              : cudaMemsetAsync(dS0, 0, nb, st));
    }
    const size_t need = kda::recurrent_bwd_workspace_bytes(N, T, H, V);
    if (workspace == nullptr || workspace_bytes < need) return KDA_ERR_INVALID_ARG;

    const size_t ntok = (size_t)N * T;
    cudaError_t e = cudaMemsetAsync(dq, 0, ntok * Hk * D * sizeof(float), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dk, 0, ntok * Hk * D * sizeof(float), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dbeta, 0, ntok * H * sizeof(float), st);
    if (e == cudaSuccess && gated)
        e = cudaMemsetAsync(dg, 0, ntok * H * (sh->gate == KDA_GATE_CHANNEL ? D : 1) * sizeof(float), st);
    if (e != cudaSuccess) return KDA_ERR_CUDA;

    kda::RecurrentBwdArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S0 = S0; a.d_out = d_out; a.d_ST = d_ST;
    a.dq = dq; a.dk = dk; a.dv = dv; a.dg = dg; a.dbeta = dbeta; a.dS0 = dS0;
    a.ws = static_cast<float*>(workspace);
    a.N = N; a.T = T; a.H = H; a.Hk = Hk; a.d_k = D; a.d_v = V; a.gate = sh->gate;
    a.scale = 1.0f / sqrtf((float)D);
    return from_cuda(kda::launch_recurrent_bwd(a, sh->dtype == KDA_BF16, st));
}

size_t kda_chunk_bwd_workspace_size(const kda_shape_t* sh, int varlen) {
    if (sh == nullptr || sh->B < 0 || sh->T < 0 || sh->H <= 0 || sh->num_seqs < 0) return 0;
    if (sh->dtype != KDA_BF16 || !tc_supports(sh->d_k, sh->d_v, sh->chunk)) return 0;
    return kda::bwd_layout(sh->B, sh->T, sh->H, sh->num_seqs, varlen != 0).bytes;
}

kda_status_t kda_chunk_bwd(const kda_shape_t* sh, const void* q, const void* k, const void* v,
                           const float* g, const float* beta, const float* S0,
                           const int32_t* cu_seqlens, const void* d_out, const float* d_ST, float* dq,
                           float* dk, float* dv, float* dg, float* dbeta, float* dS0, void* workspace,
                           size_t workspace_bytes, void* stream) {
    if (sh == nullptr) return KDA_ERR_INVALID_ARG;
    const int B = sh->B, T = sh->T, H = sh->H, N = sh->num_seqs;
    if (B < 0 || T < 0 || H <= 0 || sh->d_k <= 0 || sh->d_v <= 0 || N < 0) return KDA_ERR_INVALID_ARG;
    const int Hk = qk_heads_of(sh);
    if (Hk < 0) return KDA_ERR_INVALID_ARG;
    if (sh->dtype != KDA_F32 && sh->dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (sh->gate != KDA_GATE_CHANNEL && sh->gate != KDA_GATE_SCALAR && sh->gate != KDA_GATE_NONE)
        return KDA_ERR_INVALID_ARG;
    const bool gated = sh->gate != KDA_GATE_NONE;
    if (cu_seqlens == nullptr) {
        if (N != B) return KDA_ERR_INVALID_ARG;
    } else if (B != 1) {
        return KDA_ERR_INVALID_ARG;
    }
    const long long tok = (long long)B * T;
    // without tokens, the per-token tensors are empty (and their pointers may be null)
    if (!gated && (g != nullptr || dg != nullptr)) return KDA_ERR_INVALID_ARG;
    if (tok > 0 && (!q || !k || !v || !beta || !d_out || !dq || !dk || !dv || !dbeta || (gated && (!g || !dg))))
        return KDA_ERR_INVALID_ARG;
    const bool g_vec = sh->gate == KDA_GATE_CHANNEL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !(g_vec ? aligned16(g) : aligned4(g)) ||
        !aligned4(beta) || !aligned16(S0) || !aligned4(cu_seqlens) || !aligned16(d_out) ||
        !aligned16(d_ST) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
        !(g_vec ? aligned16(dg) : aligned4(dg)) || !aligned4(dbeta) || !aligned16(dS0))
        return KDA_ERR_MISALIGNED;
    if (sh->dtype != KDA_BF16 || !tc_supports(sh->d_k, sh->d_v, sh->chunk)) return KDA_ERR_UNSUPPORTED;
    if ((long long)N * H * 2 > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    const kda::BwdLayout bl = kda::bwd_layout(B, T, H, N, cu_seqlens != nullptr);
    if (bl.fwd.slots * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    if (workspace != nullptr) {
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_MISALIGNED;
        if (workspace_bytes < bl.bytes) return KDA_ERR_INVALID_ARG;
    }
    if (N == 0) return KDA_OK;

    kda::ChunkBwdArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S0 = S0; a.cu_seqlens = cu_seqlens;
    a.d_out = d_out; a.d_ST = d_ST;
    a.dq = dq; a.dk = dk; a.dv = dv; a.dg = dg; a.dbeta = dbeta; a.dS0 = dS0;
    a.dev_status = sh->dev_status;
    a.B = B; a.T = T; a.H = H; a.Hk = Hk; a.num_seqs = N; a.gate = sh->gate;
    a.scale = 1.0f / sqrtf((float)sh->d_k);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (Hk != H && tok > 0) {   // query/key heads shared by several value heads: summed with atomics
        e = cudaMemsetAsync(dq, 0, (size_t)tok * Hk * sh->d_k * sizeof(float), st);
        if (e == cudaSuccess) e = cudaMemsetAsync(dk, 0, (size_t)tok * Hk * sh->d_k * sizeof(float), st);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const bool pooled = ws == nullptr;
    if (pooled && cudaMallocAsync(reinterpret_cast<void**>(&ws), bl.bytes, st) != cudaSuccess) return KDA_ERR_CUDA;
    const kda::ChunkArgs fa = kda::forward_args(a);
    e = kda::launch_chunk_wy(fa, ws, bl.fwd, st);
    if (e == cudaSuccess) e = kda::launch_chunk_scans_bwd(a, ws, bl, st);
    if (e == cudaSuccess) e = kda::launch_chunk_bwd_grad(a, ws, bl, st);
    if (pooled) {
        const cudaError_t f = cudaFreeAsync(ws, st);
        if (e == cudaSuccess) e = f;
    }
    return from_cuda(e);
}

kda_status_t kda_decode_step(const kda_shape_t* sh, const void* q, const void* k, const void* v,
                             const float* g, const float* beta, float* S, void* out,
                             void* stream) {
    if (sh == nullptr) return KDA_ERR_INVALID_ARG;
    const int N = sh->B, H = sh->H, D = sh->d_k, V = sh->d_v;
    if (N < 0 || H <= 0 || D <= 0 || V <= 0 || sh->T != 1) return KDA_ERR_INVALID_ARG;
    const int Hk = qk_heads_of(sh);
    if (Hk < 0) return KDA_ERR_INVALID_ARG;
    if (sh->dtype != KDA_F32 && sh->dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (sh->gate != KDA_GATE_CHANNEL && sh->gate != KDA_GATE_SCALAR && sh->gate != KDA_GATE_NONE)
        return KDA_ERR_INVALID_ARG;
    if ((sh->gate == KDA_GATE_NONE) != (g == nullptr)) return KDA_ERR_INVALID_ARG;
    if (N > 0 && (!q || !k || !v || !beta || !S || !out)) return KDA_ERR_INVALID_ARG;
    const bool g_vec = sh->gate == KDA_GATE_CHANNEL;
    if (!aligned16(q) || !aligned16(k) || !aligned4(v) || !(g_vec ? aligned16(g) : aligned4(g)) ||
        !aligned4(beta) || !aligned16(S) || !aligned4(out))
        return KDA_ERR_MISALIGNED;
    if (D != 128 || V > 65535 * 128) return KDA_ERR_UNSUPPORTED;
    if ((long long)N * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    if (N == 0) return KDA_OK;

    kda::DecodeArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S = S; a.out = out;
    a.N = N; a.H = H; a.d_k = D; a.d_v = V; a.gate = sh->gate;
    a.Hk = Hk;
    a.scale = 1.0f / sqrtf((float)D);
    return from_cuda(kda::launch_decode(a, sh->dtype == KDA_BF16, static_cast<cudaStream_t>(stream)));
}

kda_status_t kda_selftest_bounded_wait(int32_t* dev_status, uint32_t budget_us, int32_t complete,
                                       void* stream) {
    if (dev_status == nullptr || !aligned4(dev_status)) return KDA_ERR_INVALID_ARG;
    if (budget_us < 1u || budget_us > 1000000u) return KDA_ERR_INVALID_ARG;
    return from_cuda(kda::launch_selftest_wait(dev_status, 1000ull * budget_us, complete != 0,
                                               static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
