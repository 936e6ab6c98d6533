// kda_chunk_scan.cu -- the state-scan kernel of the tensor-core prefill (its
// device code, and the design, are in kda_chunk_scan.cuh).
#include "kda_chunk_scan.cuh"

namespace kda {
namespace {

template <int NW>
__global__ void __launch_bounds__(Cfg<NW>::NT, 1) kda_chunk_scan_kernel(const __grid_constant__ ScanParams p) {
    scan_cta<NW>(p, blockIdx.x);
}

template <int NW>
cudaError_t launch_scan(const ScanParams& p, long long pairs, cudaStream_t st) {
    using G = Cfg<NW>;
    cudaError_t e = cudaFuncSetAttribute(kda_chunk_scan_kernel<NW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         G::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    return launch_after(kda_chunk_scan_kernel<NW>, dim3((unsigned)pairs), G::NT, G::SMEM_BYTES, st, p);
}

}  // namespace

cudaError_t launch_chunk_scan(const ChunkArgs& a, const uint8_t* ws, const rec::Layout& lay, cudaStream_t st,
                              float* S_chk) {
    ScanParams p;
    p.S_chk = S_chk;
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
    const long long pairs = (long long)a.num_seqs * a.H;
    return launch_scan<16>(p, pairs, st);
}

}  // namespace kda
