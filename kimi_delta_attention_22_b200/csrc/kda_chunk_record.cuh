// kda_chunk_record.cuh -- the per-(chunk, head) record through which the
// two-kernel tensor-core prefill passes its state-independent operands, and
// the workspace that holds the records.
//
// The WY kernel (kda_chunk_wy.cu) turns one chunk of one head into the
// operands of the chunkwise form that do not depend on the incoming state
// ("Chunkwise KDA" of the GeekNews summary of "You could have come up with
// Kimi Delta Attention"; the WY/UT pseudo-values of the curriculum page):
//
//   W   = T diag(beta) (K e^{Gamma})          U = T diag(beta) V
//   Qg  = Q~ e^{Gamma}                        Kd = K e^{Gamma_last - Gamma}
//   Aqk = lower(Qp) (diagonal included)       dec = e^{Gamma_last}
//
// and the state-scan kernel (kda_chunk_scan.cu) walks the chunks of a
// sequence in order with the state S (d_v x d_k, row v = value index):
//
//   E^T = U^T - S W^T,   O^T = S Qg^T + E^T Aqk^T,   S <- S Diag(dec) + E^T Kd.
//
// Every matrix is stored in fp16 (11 significant bits; every value here is
// bounded: |K e^{Gamma}|, |Kd| <= |k|, and W, U, Qg, Aqk are products of bounded
// factors) as the exact byte image of a tcgen05 shared-memory operand of the
// scan's MMAs (128-byte swizzle), so the scan kernel moves a whole record with
// one bulk copy.  Rows of a short final chunk beyond its length are zero.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace kda {
namespace rec {

constexpr int C = 64, DK = 128, DV = 128;

// Byte offsets inside one record.
constexpr int WQ = 0;        // 32 KB: rows 0-63 W, rows 64-127 Qg; (row r, channel c) at
                             //        mnmaj_off(c, r, 128) (K-major over the channel, 8-row
                             //        groups 2048 bytes apart): B operand of S [W ; Qg]^T
constexpr int KD = 32768;    // 16 KB: Kd, (token j, channel c) at mnmaj_off(c, j, 128):
                             //        MN-major B operand of E^T Kd
constexpr int AQ = 49152;    //  8 KB: Aqk, (token i, token j) at kmaj_off(i, j, 64):
                             //        K-major B operand of E^T Aqk^T
constexpr int UT = 57344;    // 16 KB: U^T, (value v, token j) at kmaj_off(v, j, 128): read
                             //        by the thread that owns value row v
constexpr int DEC = 73728;   // 512 B: fp32 dec[c]
constexpr int BYTES = 74240;
static_assert(BYTES % 256 == 0, "records must keep 256-byte alignment");

// Workspace: [slow-job list: int32 count + one entry per (slot, head)]
//            [chunk offsets: int32 per sequence + 1 (varlen only)]
//            [records: slot-major, head-minor]
// A "slot" numbers the chunks of all sequences in order: dense batches have
// ceil(T / C) slots per sequence; packed batches at most ceil(T / C) + num_seqs.
struct Layout {
    long long slots;
    size_t list_off, coff_off, rec_off, bytes;
};

inline size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

inline Layout layout(int B, int T, int H, int num_seqs, bool varlen) {
    Layout l;
    const long long nc = ((long long)T + C - 1) / C;
    l.slots = varlen ? nc + num_seqs : (long long)B * nc;
    l.list_off = 0;
    l.coff_off = round256(sizeof(int32_t) * (size_t)(1 + l.slots * H));
    l.rec_off = l.coff_off + (varlen ? round256(sizeof(int32_t) * (size_t)(num_seqs + 1)) : 0);
    l.bytes = l.rec_off + (size_t)l.slots * H * BYTES;
    return l;
}

}  // namespace rec
}  // namespace kda
