/*
 * qem.h -- C ABI of the B200-native paired-count resident (libqem.so).
 *
 * A 4D-STEM count acquisition (scan_row, scan_col, det_row, det_col), uint8 or
 * uint16, is held on the GPU entropy-coded as per-pixel 512-scan pair-tANS
 * streams (bitstream spec "qem-pair-v2") and queried without a dense copy.
 * Source: page "Paired-count resident layout" (quantem.gpu developer docs),
 * sections "Operation pipeline" (steps 1-6), "Contract" and "Verification".
 *
 * Conventions for every call:
 *  - Pointers named d_* are DEVICE pointers on the current CUDA device, h_*
 *    are HOST pointers.  The caller owns every buffer it passes; the library
 *    never frees or retains them past the call (stream-ordered: device inputs
 *    must stay valid until the work queued on `stream` has run).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *  - The resident owns all of its own device memory (payload arenas, group
 *    tables, query scratch, per-stride baselines) and releases it in qem_free.
 *  - Every call returns a qem_status.  No call falls back to the CPU; a
 *    missing or failing device returns QEM_ERR_CUDA.
 *  - Layouts: counts are row-major [scans][pixels] with scan index
 *    s = scan_row*scan_cols + scan_col and pixel p = det_row*det_cols + det_col;
 *    masks and validity maps are uint8 [pixels] (nonzero = selected / valid).
 */
#ifndef QEM_H
#define QEM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QEM_SCANS_PER_BLOCK 512

typedef enum {
    QEM_OK = 0,
    QEM_ERR_ARG = 1,        /* invalid argument (sizes, dtype, stride, out_bits)    */
    QEM_ERR_MALFORMED = 2,  /* a decoded stream failed a qem-pair-v2 check: the
                               query's output is not a result (page "Contract":
                               malformed stream -> error, the result is not returned) */
    QEM_ERR_CUDA = 3,       /* a CUDA runtime call failed                            */
    QEM_ERR_OOM = 4,        /* device allocation failed                              */
    QEM_ERR_TIMEOUT = 5,    /* a bounded wait ran out (host on the device, or a
                               kernel on its shared-memory table copy)             */
    QEM_ERR_TAINTED = 6,    /* delta refused: the stride's baseline was invalidated by
                               a failed decode (page "Contract", queued queries)      */
    QEM_ERR_STATE = 7       /* call not valid in the resident's current state         */
} qem_status;

typedef struct qem_resident qem_resident;   /* opaque */

/* Resident statistics (qem_info). */
typedef struct {
    int64_t scan_rows, scan_cols;
    int32_t det_rows, det_cols;
    int32_t dtype_bits;
    int32_t n_pixels, n_valid;
    int32_t out_bits_auto;          /* 32 or 64, the page's full-detector rule        */
    int64_t n_blocks;               /* 512-scan blocks in the acquisition              */
    int64_t n_blocks_encoded;       /* blocks appended so far                          */
    uint64_t payload_bytes;         /* encoded stream bytes                            */
    uint64_t group_bytes;           /* grouped-offset tables (68 B per 32 streams)     */
    uint64_t device_bytes;          /* all device memory the resident holds            */
    uint64_t form_count[5];         /* streams per form: empty, constant, sparse, paired, literal */
    uint64_t model_count[32];       /* paired streams per model                        */
    int32_t n_arenas;               /* payload allocations                             */
    int32_t index_leaves;           /* interaction index: leaves (0 = no index)        */
    int32_t index_roots;            /* interaction index: roots                        */
    uint64_t index_bytes;           /* interaction index: stored sums                  */
} qem_info_t;

/* Per-kernel device time, gathered with CUDA events on the launching stream
 * while profiling is enabled (qem_profile).  A masked sum launches the plan
 * and decode_reduce kernels; the slot QEM_K_FINALIZE is kept for layout and
 * stays at zero (the decode updates the kept baseline image itself). */
typedef struct {
    int64_t launches[8];
    double ms[8];
} qem_profile_t;
#define QEM_K_PLAN 0
#define QEM_K_DECODE_REDUCE 1
#define QEM_K_FINALIZE 2
#define QEM_K_DECODE_BLOCKS 3
#define QEM_K_ENC_STREAMS 4
#define QEM_K_ENC_LAYOUT 5
#define QEM_K_ENC_COMPACT 6
#define QEM_K_GENERATE 7

/* ABI string of the bitstream this library writes and reads ("qem-pair-v2").
 * Page "Contract": the coding parameters are fixed by the ABI string. */
const char *qem_abi(void);

/* Human-readable name of a qem_status. */
const char *qem_status_string(int status);

/* Create an empty resident for an acquisition of scan_rows x scan_cols scans
 * (a multiple of 512, page "Operation pipeline" step 1: complete 512-scan
 * blocks) and det_rows x det_cols pixels (1 .. 2^24-1) of dtype_bits 8 or 16.
 * d_valid: optional device uint8 [pixels] validity map (NULL = all valid);
 * copied.  Invalid pixels add nothing to sums and decode as 0 (page
 * "Contract": invalid pixels reported as zero).  Blocks are added with
 * qem_encode_append.  Errors: QEM_ERR_ARG, QEM_ERR_OOM, QEM_ERR_CUDA. */
int qem_create(int64_t scan_rows, int64_t scan_cols, int32_t det_rows, int32_t det_cols,
               int32_t dtype_bits, const uint8_t *d_valid, void *stream, qem_resident **out);

/* Encode a whole acquisition held on the device: d_counts [scans][pixels] of
 * uint8/uint16 (page "Operation pipeline" step 2: per-pixel 512-scan pair
 * streams, 1024-state tANS from 32 Poisson pair models, empty / constant /
 * sparse / incompressible forms, grouped 32-bit base + 16-bit offsets).
 * Equivalent to qem_create + qem_encode_append of every block.  Returns when
 * the resident is complete (synchronises `stream`). */
int qem_encode(const void *d_counts, int32_t dtype_bits, int64_t scan_rows, int64_t scan_cols,
               int32_t det_rows, int32_t det_cols, const uint8_t *d_valid, void *stream,
               qem_resident **out);

/* Append n_blocks complete 512-scan blocks (d_counts [n_blocks*512][pixels])
 * after the blocks already encoded (page "Operation pipeline" step 1,
 * PairedCounts.append).  Synchronises `stream` once per call (block lengths
 * decide where the payload goes).  QEM_ERR_ARG if it would pass the
 * acquisition's block count. */
int qem_encode_append(qem_resident *res, const void *d_counts, int64_t n_blocks, void *stream);

/* Masked sum (page "Operation pipeline" step 4): d_out[r][i] = sum over
 * pixels p with mask[p] && valid[p] of the count at scan 512*(r*k) + i, for
 * r = 0 .. ceil(n_blocks/k)-1 (block_stride k >= 1 touches exactly
 * ceil(blocks/k) blocks).  d_mask: device uint8 [pixels].  out_bits: 0 = auto
 * (uint32, or uint64 when a full-detector sum could exceed 2^32, page
 * "Contract"), 64 = force uint64, 32 = uint32 (QEM_ERR_ARG if auto would
 * choose 64).  d_out: caller-owned, 16-byte aligned device array of
 * ceil(B/k)*512 elements of the chosen width; *out_bits_used (may be NULL) receives 32 or 64.
 * The mask and image become this stride's baseline for qem_masked_sum_delta.
 * wait != 0: synchronise and return QEM_ERR_MALFORMED if any decoded stream
 * failed a check (d_out is then not a result).  wait == 0: return once
 * queued; errors surface at qem_finish. */
int qem_masked_sum(qem_resident *res, const uint8_t *d_mask, int32_t block_stride,
                   int32_t out_bits, void *d_out, int32_t *out_bits_used, int32_t wait,
                   void *stream);

/* Incremental masked sum (page "Operation pipeline" step 4: decode only the
 * mask difference; the baseline is kept per stride): d_out = baseline image
 * + sum over pixels entering the mask - sum over pixels leaving it, which
 * equals qem_masked_sum(d_new_mask).  With no baseline for this stride (or a
 * different output width) it runs a full query.  QEM_ERR_TAINTED when the
 * stride's baseline was invalidated by a failed decode (page "Contract",
 * queued queries); a full qem_masked_sum clears that.  Same d_out, out_bits,
 * wait rules as qem_masked_sum. */
int qem_masked_sum_delta(qem_resident *res, const uint8_t *d_new_mask, int32_t block_stride,
                         int32_t out_bits, void *d_out, int32_t *out_bits_used, int32_t wait,
                         void *stream);

/* Masked sum by complement (page "Backend Optimization Matrix", CUDA
 * checkpoint rows: dense dark field as a cached total minus the complement):
 * d_out = T - (sum over the valid pixels outside the mask), where T is the
 * resident's cached full-detector image (every valid pixel's stream decoded
 * once, on the first call, which synchronises `stream` and allocates
 * B x 512 x 8 bytes, kept until qem_free).  The result equals
 * qem_masked_sum(d_mask); it decodes the complement's streams instead of the
 * mask's, so it is the cheaper query for a mask covering most of the
 * detector.  It does not use the interaction index.  The mask and image become
 * this stride's delta baseline.  Same d_mask, block_stride, out_bits, d_out
 * and wait rules as qem_masked_sum; QEM_ERR_MALFORMED (no cache kept) if a
 * stream failed a check while the total was built. */
int qem_masked_sum_complement(qem_resident *res, const uint8_t *d_mask, int32_t block_stride,
                              int32_t out_bits, void *d_out, int32_t *out_bits_used, int32_t wait,
                              void *stream);

/* Block decode (page "Operation pipeline" step 6, decode_blocks(first,
 * scans), read as first block and block count): d_out [n_blocks*512][pixels]
 * in the native dtype (aligned to it), invalid pixels 0.  Same wait rule as the queries. */
int qem_decode_blocks(qem_resident *res, int64_t first_block, int64_t n_blocks, void *d_out,
                      int32_t wait, void *stream);

/* Scan-range decode (page "Paired-count resident layout", "Source map":
 * the decode_range and frame kernels; "Contract": queued queries,
 * session.frame(..., wait=False); "Verification": every frame compared with
 * direct sums): d_out [n_scans][pixels] in the native dtype (aligned to it)
 * receives the counts of scans first_scan .. first_scan + n_scans - 1 (scan
 * index s = scan_row * scan_cols + scan_col), invalid pixels 0; a single
 * diffraction frame is n_scans = 1.  The range may cross block boundaries
 * and must lie inside the blocks encoded so far (QEM_ERR_ARG otherwise).
 * Each stream is decoded only up to the last pair the range needs, so its
 * end-of-stream checks (final tANS state, exact section length) are left to
 * block decodes and queries; everything read is checked (header, fields,
 * form lengths, sparse order, value range, no read past the stream's
 * extent) and a failed check gives QEM_ERR_MALFORMED.  Same wait rule as
 * qem_decode_blocks (wait == 0: errors surface at qem_finish).  Profiled
 * under QEM_K_DECODE_BLOCKS. */
int qem_decode_range(qem_resident *res, int64_t first_scan, int64_t n_scans, void *d_out, int32_t wait,
                     void *stream);

/* Interaction index (page "Operation pipeline" step 3: exact per-scan sums of
 * radial-angular pixel groups, 64-pixel leaves and 16-leaf roots; step 4: a
 * mask, or its difference from the previous mask, is decomposed into index
 * groups plus residual pixels).  Builds the index of a complete resident by
 * decoding every stream once: the valid pixels are split into 16 angular
 * sectors about (center_row, center_col) (detector pixel coordinates, may be
 * fractional), sorted by distance inside each sector and cut into leaves of
 * 64; 16 consecutive leaves of a sector form a root.  For every block and
 * group the 512 sums are kept at 1, 2 or 4 bytes each (the smallest that
 * holds the group's largest sum in that block; none when all are zero).
 * Afterwards every full masked sum (any stride) takes whole groups from the
 * index and decodes only the remaining pixels; a delta decodes its changed
 * pixels (an edge that moves rarely fills a whole group); results are
 * unchanged (exact).  Rebuilding replaces the index; it synchronises
 * `stream` first.  Errors: QEM_ERR_ARG (null resident, centre not finite),
 * QEM_ERR_STATE (resident not complete), QEM_ERR_MALFORMED (a stream failed
 * its checks while summing; no index is kept), QEM_ERR_OOM, QEM_ERR_CUDA. */
int qem_build_index(qem_resident *res, double center_row, double center_col, void *stream);

/* Discard the interaction index (queries decode every masked pixel again).
 * Synchronises `stream` first. */
int qem_drop_index(qem_resident *res, void *stream);

/* The polar layout qem_build_index would use for this geometry, computed on
 * the host only (no device work): arguments and outputs as for
 * qem_index_layout; h_valid (host, n_pixels bytes, may be NULL = all valid).
 * Call once with h_slots and h_root_leaf0 NULL to learn the sizes.
 * QEM_ERR_ARG for an empty or too large detector or a non-finite centre. */
int qem_polar_layout(int32_t det_rows, int32_t det_cols, const uint8_t *h_valid, double center_row,
                     double center_col, uint32_t *h_slots, int32_t *h_root_leaf0, int32_t *n_leaves,
                     int32_t *n_roots);

/* The index's polar layout, for inspection: *n_leaves and *n_roots (may be
 * NULL); h_slots (host, may be NULL) receives 64 pixel indices per leaf, in
 * leaf order, with n_pixels marking unused slots of a sector's last leaf;
 * h_root_leaf0 (host, may be NULL) receives n_roots + 1 entries, root r
 * holding leaves [h_root_leaf0[r], h_root_leaf0[r + 1]).  QEM_ERR_STATE when
 * the resident has no index. */
int qem_index_layout(const qem_resident *res, uint32_t *h_slots, int32_t *h_root_leaf0, int32_t *n_leaves,
                     int32_t *n_roots);

/* The validity map the resident was created with: h_valid (host, n_pixels
 * bytes) receives 1 for valid and 0 for invalid pixels. */
int qem_export_valid(const qem_resident *res, uint8_t *h_valid);

/* Saved form (page "Contract": saved form; "Operation pipeline" step 5: the
 * resident arrays are written once and reopened with no decode).  qem_save
 * writes a complete resident to `path`: the magic "QGPUPAIR", a u32 header
 * length, a JSON header (format "qem-pair-resident-v1", the ABI string, the
 * geometry and each array's offset and length), then 4096-byte aligned arrays:
 * the validity map, the group records, the u64 block payload offsets and the
 * payload bytes.  The interaction index is not saved (qem_build_index
 * rebuilds it).  Errors: QEM_ERR_ARG (null argument, file not writable),
 * QEM_ERR_STATE (resident not complete), QEM_ERR_CUDA. */
int qem_save(const qem_resident *res, const char *path, void *stream);

/* Reopen a saved form as a new resident (*out; free with qem_free).  The
 * magic, the format and the ABI string must match this library's
 * ("reopen refuses another ABI"); sizes and offsets are checked.  The streams
 * themselves are checked when queried, as for qem_import.  Errors:
 * QEM_ERR_ARG (unreadable, truncated or foreign file), QEM_ERR_OOM,
 * QEM_ERR_CUDA. */
int qem_load(const char *path, void *stream, qem_resident **out);

/* The index's storage descriptors, for inspection and byte accounting: h_desc
 * (host) receives n_blocks x (n_leaves + n_roots) words, group g of block b at
 * [b * (n_leaves + n_roots) + g] (roots after the leaves); bits 30-31 give the
 * width of its 512 sums (0: all zero and not stored; 1, 2, 3: 1, 2, 4 bytes),
 * bits 0-29 the byte offset in the block's index storage.  QEM_ERR_STATE when
 * the resident has no index. */
int qem_index_desc(const qem_resident *res, uint32_t *h_desc);

/* Masked moments (the pages' fused CoM/DPC moment reduction: an exact
 * integer numerator and denominator before the float divide): for each
 * touched block row (blocks 0, k, 2k, ...) and scan, over the pixels with
 * mask && valid,
 *   d_out[0][row][scan] = sum x * d_weights[p]            (e.g. row offset)
 *   d_out[1][row][scan] = sum x * d_weights[n_pixels + p] (e.g. column offset)
 *   d_out[2][row][scan] = sum x
 * as int64 (caller-owned, 8-byte aligned, 3 * ceil(B/k) * 512 values).
 * d_weights: device int32 [2][n_pixels], each |w| <= 262143 (larger weights
 * give wrong sums, not a fault).  Centre of mass = d_out[0] / d_out[2];
 * a segmented DPC signal uses +-1 weights.  Every masked pixel is decoded
 * (the interaction index holds no weighted sums); stride baselines are not
 * touched.  Same wait rule and errors as qem_masked_sum. */
int qem_masked_moments(qem_resident *res, const uint8_t *d_mask, const int32_t *d_weights, int32_t block_stride,
                       int64_t *d_out, int32_t wait, void *stream);

/* Block decode plus amplitude (page "Operation pipeline" step 6: the feed's
 * "counts plus float32 sqrt amplitude"): as qem_decode_blocks into d_counts,
 * then d_amp (float32, same [n_blocks*512][pixels] shape, 4-byte aligned)
 * receives sqrtf(count) of every decoded count (correctly rounded; invalid
 * pixels 0).  Same wait rule and errors as qem_decode_blocks. */
int qem_decode_blocks_amplitude(qem_resident *res, int64_t first_block, int64_t n_blocks, void *d_counts,
                                float *d_amp, int32_t wait, void *stream);

/* Wait (bounded, ~60 s) for all queued work on `stream` and report any
 * malformed stream found since the last qem_finish (page "Contract":
 * session.finish() raises for a malformed stream).  On error every stride
 * baseline written since the last finish is tainted.  QEM_ERR_TIMEOUT if the
 * device did not finish in time. */
int qem_finish(qem_resident *res, void *stream);

/* Resident statistics; synchronises nothing (host-side bookkeeping). */
int qem_info(const qem_resident *res, qem_info_t *out);

/* Device counters since the last call: touched block rows decoded by masked
 * sums (ceil(B/k) per query) and streams decoded.  Synchronises `stream`. */
int qem_query_counters(qem_resident *res, uint64_t *rows_decoded, uint64_t *streams_decoded,
                       void *stream);

/* Enable (1) / disable (0) per-kernel CUDA-event timing; qem_profile_read
 * synchronises and returns the totals since enabling. */
int qem_profile(qem_resident *res, int32_t enable);
int qem_profile_read(qem_resident *res, qem_profile_t *out);

/* Release every device allocation of the resident (page "Operation
 * pipeline": the resident owns its arrays).  NULL is ignored. */
void qem_free(qem_resident *res);

/* ---- masked sum that allocates nothing ---- */

/* Largest detector (pixels) qem_masked_sum_noalloc accepts. */
#define QEM_NOALLOC_MAX_PIXELS 131072

/* Masked sum for callers that cannot allocate device memory while they query:
 * for example a render or acquisition thread that must never block on the
 * CUDA allocator (cudaMalloc can synchronise the device and stall it), code
 * that runs under an external memory budget which forbids new allocations
 * once set-up is over, or a host application whose allocator is owned by
 * another framework.  The source pages have no counterpart to this call.
 *
 * Same result as qem_masked_sum (same d_mask, block_stride, out_bits and
 * d_out rules; d_out is caller-owned) but this call performs no cudaMalloc,
 * cudaFree or other allocating routine.  Its working memory (the listed
 * pixels, their count and the error status, ~0.5 MB) is one fixed array in
 * the library's device globals, held by every GPU that loads the library
 * until the process exits.  Consequences:
 *  - the detector may have at most QEM_NOALLOC_MAX_PIXELS pixels, otherwise
 *    QEM_ERR_ARG is returned and nothing runs;
 *  - all calls share that array, which keeps the last call's contents (each
 *    call clears the status and counts it needs before using them): calls
 *    whose work overlaps on the GPU (other streams, other threads) race and
 *    give wrong results; serialise them;
 *  - what could allocate is done once per device when a resident is created
 *    on it (qem_create, qem_encode, qem_import, qem_load): looking up the
 *    array's device address (cudaGetSymbolAddress, which also loads the
 *    library code that holds it), loading the kernels this call launches and
 *    taking one pinned host word for its status; so even the first call on a
 *    device allocates nothing (QEM_ERR_CUDA if that set-up had failed);
 *  - the call waits (bounded, ~60 s, QEM_ERR_TIMEOUT) for its own work on
 *    `stream` and returns QEM_ERR_MALFORMED if a decoded stream failed a
 *    check;
 *  - it neither reads nor updates the per-stride delta baselines, and does not
 *    use the interaction index (results are the same with or without one).
 * The resident must live on the current device and be complete. */
int qem_masked_sum_noalloc(qem_resident *res, const uint8_t *d_mask, int32_t block_stride,
                           int32_t out_bits, void *d_out, void *stream);

/* ---- encoded form, host side (export for inspection/saving, import) ---- */

/* Payload length of block b in bytes. */
int qem_block_bytes(const qem_resident *res, int64_t block, uint64_t *nbytes);

/* Copy block b's group records (ceil(P/32) x 17 uint32, spec S1) and payload
 * bytes to host buffers; synchronises `stream`. */
int qem_export_block(const qem_resident *res, int64_t block, uint32_t *h_groups,
                     uint8_t *h_payload, void *stream);

/* Build a resident from an encoded form held on the host: h_groups
 * [n_blocks][ceil(P/32)][17] uint32, h_payload the concatenated block
 * payloads, h_block_off [n_blocks+1] byte offsets of each block in
 * h_payload.  Nothing is validated here; malformed streams surface when
 * queried.  Synchronises `stream`. */
int qem_import(int64_t scan_rows, int64_t scan_cols, int32_t det_rows, int32_t det_cols,
               int32_t dtype_bits, const uint32_t *h_groups, const uint8_t *h_payload,
               const uint64_t *h_block_off, const uint8_t *h_valid, void *stream,
               qem_resident **out);

/* Each pixel's decode class, as the query plans use it to order their work and
 * to weigh an index item against residual pixels: h_class (host, n_pixels
 * bytes) receives 1 for pixels whose block-0 stream is light (empty, sparse,
 * or paired with a low-dose model and no base or raw bits, decoded by runs)
 * and 0 for the others (decoded pair by pair).  Synchronises the device. */
int qem_pixel_classes(const qem_resident *res, uint8_t *h_class);

/* The library's own model tables (spec S4), computed on the host:
 * freq [32][256] uint16, amax [32] uint8, cost [32][16] uint32. */
int qem_model_tables(uint16_t *h_freq, uint8_t *h_amax, uint32_t *h_cost);

/* ---- synthetic input generator (bench and tests) ---- */

/* Counter-based synthetic counts for scans [scan0, scan0+n_scans):
 * z = SplitMix64 output number (s*P + p + 1) from `seed`, u = z >> 11;
 * per pixel class (d_class_desc [C][4] uint32: kind, offset, length, value):
 * kind 0 Poisson by inverse CDF, count = min{k : u < d_thresholds[offset+k]};
 * kind 1 uniform, count = z & dtype_max; kind 2 constant `value`; then
 * clipped to dtype_max.  d_out [n_scans][n_pixels]. */
int qem_generate_counts(void *d_out, int32_t dtype_bits, uint64_t seed, int64_t scan0,
                        int64_t n_scans, int32_t n_pixels, const uint32_t *d_pixel_class,
                        const uint32_t *d_class_desc, const uint64_t *d_thresholds,
                        void *stream);

#ifdef __cplusplus
}
#endif
#endif /* QEM_H */
