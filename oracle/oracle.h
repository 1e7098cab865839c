/*
 * oracle.h -- CPU oracle for the paired-count resident (qem-pair-v2).
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * bench's cpu_baseline / reference leg may load or call this code.  It shares
 * no code, header, table or constant generator with the CUDA library; both
 * follow the written bitstream specification independently.
 *
 * Source pages: "Paired-count resident layout" (quantem.gpu developer docs),
 * sections "Operation pipeline" (steps 1-6), "Contract" and "Verification".
 *
 * Every function is plain and sequential: bits are read and written one at a
 * time, tables are built by walking the specification's steps in order.
 */
#ifndef QEM_ORACLE_H
#define QEM_ORACLE_H
#include <stdint.h>
#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* error codes returned by the oracle's stream checks */
#define ORC_OK 0
#define ORC_BAD_RESERVED 1      /* reserved header bit set                     */
#define ORC_BAD_FORM 2          /* form code not in {1,2,3,4}                  */
#define ORC_BAD_FIELDS 3        /* model/shift/base fields on a non-paired form */
#define ORC_BAD_LENGTH 4        /* extent does not equal the form's length      */
#define ORC_BAD_SPARSE 5        /* sparse count/positions/values invalid        */
#define ORC_BAD_CONSTANT 6      /* constant value 0                             */
#define ORC_BAD_STATE 7         /* tANS final state != 1024 or symbol outside   */
#define ORC_BAD_PAD 8           /* nonzero pad bits                             */
#define ORC_BAD_OFFSETS 9       /* group offsets decreasing / beyond payload    */
#define ORC_BAD_MODEL 10        /* paired symbol outside the model's box        */

/* Model tables (spec section "Models").  freq[m][s], s = a + 16 b. */
void orc_models(uint16_t freq[32][256], uint8_t amax[32], uint32_t cost[32][16]);
/* Decoder table: for model m, slot i: sym, nb, newbase. */
void orc_decode_table(int m, uint8_t sym[1024], uint8_t nb[1024], uint16_t newbase[1024]);

/* Encode one 512-count stream (values in native width w = 1 or 2 bytes).
 * Writes at most 2 + 512*w bytes to out; *len = 0 means the empty form. */
void orc_encode_stream(const uint16_t v[512], int w, uint8_t *out, int *len);
/* Decode one stream of `len` bytes; fills v[512].  Returns ORC_OK or an error. */
int orc_decode_stream(const uint8_t *s, int len, int w, uint16_t v[512]);

/* Encode one 512-scan block: counts [512][P] (uint8 when w==1, uint16 when w==2).
 * groups: ceil(P/32) records of 17 uint32 (base, then 32 uint16 rel_end).
 * payload must hold (2 + 512 w) * P bytes.  Returns the block's byte length. */
uint64_t orc_encode_block(const void *counts, int w, int P, uint32_t *groups, uint8_t *payload);

/* Decode-based masked partial sum over one block:
 * out[i] += sign[j] * x[i][pix[j]] for i < 512, j < n (int64 accumulation).
 * Returns ORC_OK or the first error found; out is then unspecified. */
int orc_block_masked_sum(const uint32_t *groups, const uint8_t *payload, uint64_t len,
                         int w, int P, const int32_t *pix, const int8_t *sign, int n,
                         int64_t out[512]);

/* Decode every stream of one block into counts [512][P] (native width). */
int orc_decode_block(const uint32_t *groups, const uint8_t *payload, uint64_t len,
                     int w, int P, void *out);

/* Test introspection: exact paired length with a forced model (-1 when the
 * model's box cannot hold the stream), and the candidate sizes of a stream:
 * info = {S_sparse (2^30 when n > 256), S_paired, S_literal, selected model}. */
int orc_paired_size(const uint16_t v[512], int w, int model);
void orc_stream_sizes(const uint16_t v[512], int w, int32_t info[4]);

#ifdef __cplusplus
}
#endif
#endif
