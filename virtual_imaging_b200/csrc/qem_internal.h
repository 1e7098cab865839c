// qem_internal.h -- shared declarations of libqem's host code and kernels.
//
// Bitstream: qem-pair-v2 (page "Paired-count resident layout", "Operation
// pipeline" step 2 and "Contract"; the bit-level choices are the library's
// own written spec, sections S1-S7, cited as "spec Sn").
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qem.h"

namespace qem {

constexpr int kScans = 512;        // scans per block (page: complete 512-scan blocks)
constexpr int kPairs = 256;        // consecutive count pairs per stream
constexpr int kStates = 1024;      // tANS states (page: 1024-state table)
constexpr int kModels = 32;        // Poisson pair models (page: 32)
constexpr int kGroupWords = 17;    // 1 x u32 base + 32 x u16 relative ends (spec S1)
constexpr int kSlotWords = 84;     // per-stream tANS scratch: >= ceil((10 + 256*10)/32) + 1 words, 16-byte multiple
constexpr int kArenaPad = 64;      // zero bytes after the last block of an arena
constexpr int kRunModels = 8;      // models that may be decoded by runs (their tables replace the decode tables in shared memory)
constexpr int kOneStateModels = 8; // spec S3/S5: models 0-7 code a paired stream with one tANS state,
                                   // models 8-31 with two interleaved ones (A: even pairs, B: odd pairs)

enum Form : int { kEmpty = 0, kConstant = 1, kSparse = 2, kPaired = 3, kLiteral = 4 };

// device status flags (spec S7); any nonzero flag other than kErrWait means
// "malformed"; kErrWait: a bounded in-kernel wait ran out
enum : uint32_t {
    kErrReserved = 1u << 0,
    kErrForm = 1u << 1,
    kErrFields = 1u << 2,
    kErrLength = 1u << 3,
    kErrSparse = 1u << 4,
    kErrConstant = 1u << 5,
    kErrState = 1u << 6,
    kErrPad = 1u << 7,
    kErrOffsets = 1u << 8,
    kErrValue = 1u << 9,
    kErrWait = 1u << 31,
};

struct DevStatus {
    uint32_t flags;
    uint32_t reserved[3];
    unsigned long long rows;      // touched block rows decoded by masked sums
    unsigned long long streams;   // streams decoded by masked sums
};

// Device-resident model tables.
//  dec[m][slot]   : bits 0-9 newbase, 10-13 nb, byte 2 = hi_a, byte 3 = hi_b
//  enc_sym[m][s]  : bits 0-10 f, 11-21 cum (start of s in enc_slot), 22-25 k0 = 10 - floor(log2 f)
//  enc_slot[m][i] : slots of each symbol in ascending order, grouped by symbol
//  cost[m][v], amax[m] : selection costs and box sizes (spec S4)
struct Tables {
    const uint32_t *dec;
    const uint32_t *enc_sym;
    const uint16_t *enc_slot;
    const uint32_t *cost;
    const uint32_t *amax;
    const uint32_t *runs;     // [m < kRunModels][slot]: one run event (see HostTables::runs)
    uint32_t skip_models;     // bit m set: model m's streams are decoded by runs (a prefix of the models)
};

struct HostTables {
    uint16_t freq[kModels][256];
    uint8_t amax[kModels];
    uint32_t cost[kModels][16];
    uint32_t dec[kModels][kStates];
    uint32_t enc_sym[kModels][256];
    uint16_t enc_slot[kModels][kStates];
    // runs[m][slot], for the low-dose models m < kRunModels: from state slot,
    // r = min(63, length of the chain of zero-bit (0,0) steps starting there)
    // steps are jumped, landing on slot e; then e's ordinary decode step
    // follows.  Bits 0-9 newbase(e), 10-13 nb(e), 14-19 r, 20-23 and 24-27 the
    // two counts of e's symbol, 28: e != 0 (a stream may end on e only if e is
    // state 1024, slot 0).
    uint32_t runs[kRunModels][kStates];
    uint32_t skip_models;
};

// What the query kernels read of a resident.
struct View {
    const uint32_t *groups;               // [B][G][17]
    const unsigned long long *blk_ptr;    // [B] device address of each block's payload
    const uint32_t *blk_len;              // [B] payload bytes of each block
    const uint8_t *valid;                 // [P]
    int P;
    int G;
    int w;                                // bytes per count (1 or 2)
    long long B;
};

// Interaction index of a resident (absent when desc is null): per block, the
// 512 per-scan sums of each of G = L + R pixel groups (L leaves of at most 64
// pixels, R roots of at most 16 leaves), each group stored at one width.
struct IndexView {
    const uint32_t *desc;                 // [B][G]: bits 0-29 byte offset, 30-31 width code
    const unsigned long long *base;       // [B] device address of each block's index bytes
    const uint32_t *items;                // the query's index items (written by the plan)
    int L;
    int G;
};

const HostTables &host_tables();          // built once per process (tables.cu)

// What the allocation-free masked sum needs from a resident (api.cu).
struct ResidentQuery {
    View view;
    Tables tables;
    int P;
    long long B;
    bool complete;
    int out_bits_auto;
    int n_sm;
    int device;
    const uint8_t *valid;
    const uint8_t *pclass;        // per pixel: 1 = light streams, 0 = heavy
    void *noalloc_scratch;        // device address of the fixed working array (noalloc.cu)
    uint32_t *noalloc_flags;      // pinned host word for its status read-back
};
int resident_query_view(const qem_resident *r, ResidentQuery *q);

// Set-up of the allocation-free masked sum on the current device, run when a
// resident is created (noalloc.cu): looks up the fixed array's device address,
// loads the kernels that call uses, and keeps one pinned host word per device
// for its status.  QEM_OK or QEM_ERR_CUDA / QEM_ERR_OOM.
int noalloc_setup(int device, void **scratch, uint32_t **h_flags);

// Wait (bounded, ~60 s) until all work queued on `st` has finished, polling the
// stream itself (creates nothing).  QEM_OK, QEM_ERR_TIMEOUT or QEM_ERR_CUDA.
int bounded_stream_wait(cudaStream_t st);

// Load the decode kernels a masked sum launches (lazy module loading would
// otherwise load them at their first launch) and set their shared-memory limits.
cudaError_t preload_query_kernels();

// ---- kernel launchers (kernels.cu); all stream-ordered, return cudaError_t ----
cudaError_t launch_generate(void *out, int bits, uint64_t seed, int64_t scan0, int64_t n_scans,
                            int P, const uint32_t *pclass, const uint32_t *desc,
                            const uint64_t *thr, cudaStream_t st);

cudaError_t launch_enc_streams(const void *counts, int w, int P, int nblk, Tables tb,
                               uint4 *desc, uint32_t *slots, unsigned long long *stats,
                               uint8_t *pclass, cudaStream_t st);
cudaError_t launch_enc_layout(uint4 *desc, int P, int G, int nblk, uint32_t *groups,
                              uint32_t *blk_len, cudaStream_t st);
cudaError_t launch_enc_compact(const void *counts, int w, int P, int nblk, const uint4 *desc,
                               const uint32_t *slots, const unsigned long long *blk_dst,
                               cudaStream_t st);

// decode_reduce reads count[0] heavy entries from list[0..) and count[1]
// light entries from list[P - count[1], P).
// plan: builds the signed pixel list, heavy class from the front (count[0]),
// light class from the back (count[1]), clears count_next (the pair the next
// query uses) and initialises the rows: mode 0 = full query (out = keep = 0),
// 1 = delta (out = keep, the stride's kept image)
// 2 = complement (the valid pixels outside the mask, subtracted; out = keep =
// the rows r * stride of total, the cached full-detector image [B][512] uint64);
// keep may be null in mode 0
cudaError_t launch_plan(const uint8_t *mask, const uint8_t *valid, const uint8_t *pclass,
                        uint8_t *base_mask, int P, int mode, uint32_t *list, uint32_t *count,
                        uint32_t *count_next, void *out, void *keep, long long n_elems, int out_bytes,
                        cudaStream_t st, const unsigned long long *total = nullptr, int stride = 1);
// keep (may be null): a second image that receives the same additions as out;
// ix.desc null: no index items (count[2] is not read)
cudaError_t launch_decode_reduce(View v, Tables tb, const uint32_t *list, const uint32_t *count,
                                 int stride, long long rows, void *out, int out_bytes,
                                 DevStatus *status, int n_sm, cudaStream_t st, bool delta = false,
                                 void *keep = nullptr, IndexView ix = IndexView{nullptr, nullptr, nullptr, 0, 0},
                                 bool signed_list = false);
cudaError_t launch_amplitude(const void *counts, int w, float *amp, long long n, cudaStream_t st);
// masked moments: out int64 [3][rows][512] = (sum x*wr, sum x*wc, sum x) per scan
cudaError_t launch_moments(View v, Tables tb, const uint32_t *list, const uint32_t *count, const int32_t *weights,
                           int stride, long long rows, long long *out, DevStatus *status, cudaStream_t st);
// interaction index build (leafsum zeroed by the caller: [nblk][L][512] u32)
cudaError_t launch_index_sums(View v, Tables tb, const uint32_t *slots, int L, long long b0, int nblk,
                              uint32_t *leafsum, DevStatus *status, int n_sm, cudaStream_t st);
cudaError_t launch_index_size(const uint32_t *leafsum, const int *root_leaf0, int L, int G, int nblk, uint32_t *desc,
                              unsigned long long *total, cudaStream_t st);
cudaError_t launch_index_pack(const uint32_t *leafsum, const int *root_leaf0, int L, int G, long long b0, int nblk,
                              const uint32_t *desc_all, const unsigned long long *base, cudaStream_t st);
// plan over the polar layout: residual list + index items (count[2])
cudaError_t launch_plan_index(const uint8_t *mask, const uint8_t *pclass, uint8_t *base_mask, int P, int mode,
                              const uint32_t *slots, const int *root_leaf0, int R, uint32_t *list, uint32_t *items,
                              uint32_t *count, uint32_t *count_next, void *out, void *keep, long long n_elems,
                              int out_bytes, cudaStream_t st);
cudaError_t launch_decode_blocks(View v, Tables tb, long long first, long long n, void *out,
                                 DevStatus *status, cudaStream_t st);
// scans [first, first + n) of the acquisition into out [n][P] (native dtype)
cudaError_t launch_decode_range(View v, Tables tb, long long first, long long n, void *out, DevStatus *status,
                                cudaStream_t st);

}  // namespace qem
