/*
 * oracle.c -- plain CPU oracle for the paired-count resident (qem-pair-v2).
 *
 * TEST INFRASTRUCTURE ONLY (see oracle.h).  Nothing here is used by the CUDA
 * library; the library implements the same written specification on its own.
 *
 * Source pages: "Paired-count resident layout", section "Operation pipeline"
 * step 2 (pair streams, 1024-state tANS from 32 Poisson pair models, empty /
 * constant / sparse / incompressible forms, grouped offsets) and section
 * "Contract" (2-byte stream header, sparse preferred unless the paired stream
 * saves at least two bytes; malformed streams raise).  Where the pages leave
 * the format open, this file follows the build's own qem-pair-v2 spec, whose
 * numbered sections are cited below as "spec S<n>".
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define NSTATE 1024          /* tANS states L (pages: 1024-state table)      */
#define NMODEL 32            /* Poisson pair models (pages: 32)               */
#define NPAIR 256            /* 512 scans -> 256 consecutive count pairs      */
#define SPREAD_STEP 643      /* spec S5: odd step 5L/8 + 3                     */
#define ONE_STATE_MODELS 8   /* spec S3/S5: models 0-7 code a paired stream with one
                                tANS state; models 8-31 with two interleaved states
                                (state A for even pairs, B for odd pairs)        */

#define FORM_CONSTANT 1
#define FORM_SPARSE 2
#define FORM_PAIRED 3
#define FORM_LITERAL 4

/* ------------------------------------------------------------------------- */
/* spec S4: the 32 models                                                     */
/* ------------------------------------------------------------------------- */
typedef struct {
    int ready;
    uint16_t freq[NMODEL][256];
    uint8_t amax[NMODEL];
    uint32_t cost[NMODEL][16];
    /* spec S5: spread and tables */
    uint8_t spread[NMODEL][NSTATE];
    uint8_t dsym[NMODEL][NSTATE];
    uint8_t dnb[NMODEL][NSTATE];
    uint16_t dnewbase[NMODEL][NSTATE];
    uint16_t cum[NMODEL][257];
    uint16_t sorted_slot[NMODEL][NSTATE];
} Models;

static Models M;

static void build_model(int m)
{
    double lam = 0.005 * pow(3200.0, (double)m / 31.0);
    double q[16];
    double acc;
    int v, a, b, A;

    /* Poisson(lam) on 0..14, tail folded into 15 */
    q[0] = exp(-lam);
    for (v = 1; v < 15; v++)
        q[v] = (q[v - 1] * lam) / (double)v;
    acc = 0.0;
    for (v = 0; v < 15; v++)
        acc += q[v];
    q[15] = 1.0 - acc;
    if (q[15] < 0.0)
        q[15] = 0.0;

    /* box: smallest A whose tail beyond A is below 2^-20 */
    for (A = 0; A < 15; A++) {
        double tail = 0.0;
        for (v = A + 1; v < 16; v++)
            tail += q[v];
        if (tail < 1.0 / 1048576.0)
            break;
    }
    M.amax[m] = (uint8_t)A;

    /* element pmf renormalised over the box */
    double S = 0.0, t[16];
    for (v = 0; v <= A; v++)
        S += q[v];
    for (v = 0; v < 16; v++)
        t[v] = (v <= A) ? q[v] / S : 0.0;

    /* selection costs: round(256 * -log2 t_v) for v in the box */
    for (v = 0; v < 16; v++)
        M.cost[m][v] = (v <= A) ? (uint32_t)floor(-256.0 * log2(t[v]) + 0.5) : 0xFFFFFFFFu;

    /* quantise the product pmf: one slot per box symbol, then floor of the
     * rest, then largest fractional parts (ties to the lower symbol) */
    int nbox = (A + 1) * (A + 1);
    int K = NSTATE - nbox;
    double raw[256], frac[256];
    int sum = 0, s;
    memset(M.freq[m], 0, sizeof(M.freq[m]));
    for (s = 0; s < 256; s++) {
        a = s & 15;
        b = s >> 4;
        if (a > A || b > A) {
            raw[s] = 0.0;
            frac[s] = -1.0;
            continue;
        }
        raw[s] = (t[a] * t[b]) * (double)K;
        double fl = floor(raw[s]);
        frac[s] = raw[s] - fl;
        M.freq[m][s] = (uint16_t)(1 + (int)fl);
        sum += M.freq[m][s];
    }
    int R = NSTATE - sum;
    while (R-- > 0) {
        int best = -1;
        for (s = 0; s < 256; s++)
            if (frac[s] >= 0.0 && (best < 0 || frac[s] > frac[best]))
                best = s;
        M.freq[m][best] += 1;
        frac[best] = -1.0;
    }

    /* spread: walk the slots with an odd step, symbols in ascending order */
    int pos = 0, r;
    for (s = 0; s < 256; s++)
        for (r = 0; r < M.freq[m][s]; r++) {
            M.spread[m][pos] = (uint8_t)s;
            pos = (pos + SPREAD_STEP) & (NSTATE - 1);
        }

    /* decode entries: the t-th slot (ascending) of symbol s has y = f + t */
    int occ[256];
    memset(occ, 0, sizeof(occ));
    M.cum[m][0] = 0;
    for (s = 0; s < 256; s++)
        M.cum[m][s + 1] = (uint16_t)(M.cum[m][s] + M.freq[m][s]);
    for (int i = 0; i < NSTATE; i++) {
        s = M.spread[m][i];
        int f = M.freq[m][s];
        int y = f + occ[s];
        M.sorted_slot[m][M.cum[m][s] + occ[s]] = (uint16_t)i;
        occ[s]++;
        int lg = 0;
        while ((2 << lg) <= y)
            lg++;                          /* lg = floor(log2 y) */
        int nb = 10 - lg;
        M.dsym[m][i] = (uint8_t)s;
        M.dnb[m][i] = (uint8_t)nb;
        M.dnewbase[m][i] = (uint16_t)((y << nb) - NSTATE);
    }
}

static void ensure_models(void)
{
    if (M.ready)
        return;
    for (int m = 0; m < NMODEL; m++)
        build_model(m);
    M.ready = 1;
}

void orc_models(uint16_t freq[32][256], uint8_t amax[32], uint32_t cost[32][16])
{
    ensure_models();
    memcpy(freq, M.freq, sizeof(M.freq));
    memcpy(amax, M.amax, sizeof(M.amax));
    memcpy(cost, M.cost, sizeof(M.cost));
}

void orc_decode_table(int m, uint8_t sym[1024], uint8_t nb[1024], uint16_t newbase[1024])
{
    ensure_models();
    memcpy(sym, M.dsym[m], NSTATE);
    memcpy(nb, M.dnb[m], NSTATE);
    memcpy(newbase, M.dnewbase[m], NSTATE * sizeof(uint16_t));
}

/* ------------------------------------------------------------------------- */
/* bit I/O, one bit at a time, LSB-first within each byte (spec S3)          */
/* ------------------------------------------------------------------------- */
static void put_bits(uint8_t *buf, long *pos, uint32_t value, int n)
{
    for (int i = 0; i < n; i++) {
        if ((value >> i) & 1u)
            buf[*pos >> 3] |= (uint8_t)(1u << (*pos & 7));
        (*pos)++;
    }
}

/* returns -1 when the read would pass `limit` bits */
static long get_bits(const uint8_t *buf, long *pos, int n, long limit)
{
    long v = 0;
    if (*pos + n > limit)
        return -1;
    for (int i = 0; i < n; i++) {
        if ((buf[*pos >> 3] >> (*pos & 7)) & 1u)
            v |= 1L << i;
        (*pos)++;
    }
    return v;
}

static void put_native(uint8_t *p, int w, uint32_t v)
{
    p[0] = (uint8_t)(v & 0xFF);
    if (w == 2)
        p[1] = (uint8_t)(v >> 8);
}

static uint32_t get_native(const uint8_t *p, int w)
{
    return w == 2 ? (uint32_t)p[0] | ((uint32_t)p[1] << 8) : (uint32_t)p[0];
}

static int bitlen(uint32_t x)
{
    int n = 0;
    while (x) {
        n++;
        x >>= 1;
    }
    return n;
}

/* ------------------------------------------------------------------------- */
/* spec S6: the encoder                                                       */
/* ------------------------------------------------------------------------- */

/* spec S3 paired form; returns its length, writes it to out (zeroed first).
 * force_model >= 0 codes with that model instead of selecting one (returns -1
 * when the model's box cannot hold the stream); *model_out gets the model. */
static int encode_paired(const uint16_t v[512], int w, uint8_t *out, int force_model, int *model_out)
{
    uint32_t mn = 0xFFFFFFFFu, mx = 0;
    int e, j;
    for (e = 0; e < 512; e++) {
        if (v[e] < mn) mn = v[e];
        if (v[e] > mx) mx = v[e];
    }
    int has_base = mn > 0;
    uint32_t base = has_base ? mn : 0;
    int shift = bitlen(mx - base) - 4;
    if (shift < 0)
        shift = 0;

    uint32_t hi[512], lo[512];
    for (e = 0; e < 512; e++) {
        hi[e] = (v[e] - base) >> shift;
        lo[e] = (v[e] - base) & ((1u << shift) - 1u);
    }

    /* model: lowest fixed-point cost among models whose box holds every hi */
    uint32_t maxhi = 0, h[16];
    memset(h, 0, sizeof(h));
    for (e = 0; e < 512; e++) {
        h[hi[e]]++;
        if (hi[e] > maxhi) maxhi = hi[e];
    }
    int model = -1;
    uint64_t best = 0;
    if (force_model >= 0) {
        if (M.amax[force_model] < maxhi)
            return -1;
        model = force_model;
    }
    for (int m = 0; m < NMODEL && force_model < 0; m++) {
        if (M.amax[m] < maxhi)
            continue;
        uint64_t c = 0;
        for (int k = 0; k <= (int)maxhi; k++)
            c += (uint64_t)h[k] * M.cost[m][k];
        if (model < 0 || c < best) {
            model = m;
            best = c;
        }
    }

    /* tANS over pairs 255..0, every state starting from 1024; with two states,
       pair j is coded on state j & 1 */
    uint32_t chunk_v[NPAIR];
    int chunk_n[NPAIR];
    int two = model >= ONE_STATE_MODELS;
    uint32_t X[2] = {NSTATE, NSTATE};
    for (j = NPAIR - 1; j >= 0; j--) {
        int q = two ? (j & 1) : 0;
        int s = (int)(hi[2 * j] + 16u * hi[2 * j + 1]);
        uint32_t f = M.freq[model][s];
        int k = 0;
        while ((X[q] >> k) >= 2 * f)
            k++;
        chunk_v[j] = X[q] & ((1u << k) - 1u);
        chunk_n[j] = k;
        uint32_t y = X[q] >> k;
        X[q] = NSTATE + M.sorted_slot[model][M.cum[model][s] + (y - f)];
    }

    *model_out = model;
    int hdr = FORM_PAIRED | (model << 3) | (shift << 8) | (has_base << 12);
    long pos;
    int off = 2;
    out[0] = (uint8_t)(hdr & 0xFF);
    out[1] = (uint8_t)(hdr >> 8);
    if (has_base) {
        put_native(out + off, w, base);
        off += w;
    }
    pos = 0;
    for (e = 0; e < 512; e++)
        put_bits(out + off, &pos, lo[e], shift);
    off += 64 * shift;
    pos = 0;
    put_bits(out + off, &pos, X[0] - NSTATE, 10);
    if (two)
        put_bits(out + off, &pos, X[1] - NSTATE, 10);
    for (j = 0; j < NPAIR; j++)
        put_bits(out + off, &pos, chunk_v[j], chunk_n[j]);
    return off + (int)((pos + 7) / 8);
}

void orc_encode_stream(const uint16_t v[512], int w, uint8_t *out, int *len)
{
    ensure_models();
    int e, n = 0;
    uint32_t mn = 0xFFFFFFFFu, mx = 0;
    for (e = 0; e < 512; e++) {
        if (v[e]) n++;
        if (v[e] < mn) mn = v[e];
        if (v[e] > mx) mx = v[e];
    }
    if (n == 0) {                                   /* empty: zero-length extent */
        *len = 0;
        return;
    }
    if (mn == mx) {                                 /* constant */
        out[0] = FORM_CONSTANT;
        out[1] = 0;
        put_native(out + 2, w, mn);
        *len = 2 + w;
        return;
    }
    int s_lit = 2 + 512 * w;
    int s_sparse = n <= 256 ? 3 + (9 * n + 7) / 8 + n * w : 1 << 30;
    uint8_t paired[2 + 2 + 64 * 12 + 332];
    memset(paired, 0, sizeof(paired));
    int model;
    int s_paired = encode_paired(v, w, paired, -1, &model);

    int form, size;
    if (s_sparse <= s_paired + 1) {
        form = FORM_SPARSE;
        size = s_sparse;
    } else {
        form = FORM_PAIRED;
        size = s_paired;
    }
    if (size >= s_lit)
        form = FORM_LITERAL;

    memset(out, 0, (size_t)s_lit);
    if (form == FORM_PAIRED) {
        memcpy(out, paired, (size_t)s_paired);
        *len = s_paired;
    } else if (form == FORM_SPARSE) {
        long pos = 0;
        int k = 0;
        out[0] = FORM_SPARSE;
        out[1] = 0;
        out[2] = (uint8_t)(n - 1);
        for (e = 0; e < 512; e++)
            if (v[e])
                put_bits(out + 3, &pos, (uint32_t)e, 9);
        int voff = 3 + (9 * n + 7) / 8;
        for (e = 0; e < 512; e++)
            if (v[e]) {
                put_native(out + voff + k * w, w, v[e]);
                k++;
            }
        *len = s_sparse;
    } else {
        out[0] = FORM_LITERAL;
        out[1] = 0;
        for (e = 0; e < 512; e++)
            put_native(out + 2 + e * w, w, v[e]);
        *len = s_lit;
    }
}

/* ------------------------------------------------------------------------- */
/* spec S3 / S7: the decoder with every malformed-stream check                */
/* ------------------------------------------------------------------------- */
int orc_decode_stream(const uint8_t *s, int len, int w, uint16_t v[512])
{
    ensure_models();
    uint32_t dmax = (w == 2) ? 0xFFFFu : 0xFFu;
    int e, j;
    if (len == 0) {
        for (e = 0; e < 512; e++)
            v[e] = 0;
        return ORC_OK;
    }
    if (len < 2)
        return ORC_BAD_LENGTH;
    uint32_t hdr = (uint32_t)s[0] | ((uint32_t)s[1] << 8);
    if (hdr >> 13)
        return ORC_BAD_RESERVED;
    int form = (int)(hdr & 7), model = (int)((hdr >> 3) & 31);
    int shift = (int)((hdr >> 8) & 15), has_base = (int)((hdr >> 12) & 1);
    if (form < FORM_CONSTANT || form > FORM_LITERAL)
        return ORC_BAD_FORM;
    if (form != FORM_PAIRED && (model || shift || has_base))
        return ORC_BAD_FIELDS;

    if (form == FORM_CONSTANT) {
        if (len != 2 + w)
            return ORC_BAD_LENGTH;
        uint32_t c = get_native(s + 2, w);
        if (c == 0)
            return ORC_BAD_CONSTANT;
        for (e = 0; e < 512; e++)
            v[e] = (uint16_t)c;
        return ORC_OK;
    }
    if (form == FORM_LITERAL) {
        if (len != 2 + 512 * w)
            return ORC_BAD_LENGTH;
        for (e = 0; e < 512; e++)
            v[e] = (uint16_t)get_native(s + 2 + e * w, w);
        return ORC_OK;
    }
    if (form == FORM_SPARSE) {
        if (len < 3)
            return ORC_BAD_LENGTH;
        int n = s[2] + 1;
        int pbytes = (9 * n + 7) / 8;
        if (len != 3 + pbytes + n * w)
            return ORC_BAD_LENGTH;
        for (e = 0; e < 512; e++)
            v[e] = 0;
        long pos = 0, limit = 8L * pbytes;
        long prev = -1;
        for (int k = 0; k < n; k++) {
            long p = get_bits(s + 3, &pos, 9, limit);
            if (p <= prev)
                return ORC_BAD_SPARSE;
            prev = p;
            uint32_t val = get_native(s + 3 + pbytes + k * w, w);
            if (val == 0)
                return ORC_BAD_SPARSE;
            v[p] = (uint16_t)val;
        }
        while (pos < limit)
            if (get_bits(s + 3, &pos, 1, limit) != 0)
                return ORC_BAD_PAD;
        return ORC_OK;
    }

    /* paired */
    if (shift > 8 * w - 4)
        return ORC_BAD_FIELDS;
    int off = 2;
    uint32_t base = 0;
    if (has_base) {
        if (len < off + w)
            return ORC_BAD_LENGTH;
        base = get_native(s + off, w);
        off += w;
    }
    int raw_off = off;
    off += 64 * shift;
    if (len < off + 2)
        return ORC_BAD_LENGTH;
    const uint8_t *ts = s + off;
    long limit = 8L * (len - off);
    long pos = 0;
    int two = model >= ONE_STATE_MODELS;
    uint32_t X[2] = {NSTATE, NSTATE};
    for (int q = 0; q < 1 + two; q++) {
        long x0 = get_bits(ts, &pos, 10, limit);
        if (x0 < 0)
            return ORC_BAD_LENGTH;
        X[q] = NSTATE + (uint32_t)x0;
    }
    uint32_t hi[512];
    for (j = 0; j < NPAIR; j++) {
        int q = two ? (j & 1) : 0;
        int slot = (int)(X[q] - NSTATE);
        int sym = M.dsym[model][slot];
        int nb = M.dnb[model][slot];
        long bits = get_bits(ts, &pos, nb, limit);
        if (bits < 0)
            return ORC_BAD_LENGTH;
        hi[2 * j] = (uint32_t)(sym & 15);
        hi[2 * j + 1] = (uint32_t)(sym >> 4);
        X[q] = NSTATE + M.dnewbase[model][slot] + (uint32_t)bits;
    }
    if (X[0] != NSTATE || X[1] != NSTATE)
        return ORC_BAD_STATE;
    if ((pos + 7) / 8 != len - off)
        return ORC_BAD_LENGTH;
    while (pos < limit)
        if (get_bits(ts, &pos, 1, limit) != 0)
            return ORC_BAD_PAD;
    long rpos = 0;
    for (e = 0; e < 512; e++) {
        long lo = get_bits(s + raw_off, &rpos, shift, 8L * 64 * shift);
        uint32_t val = base + ((hi[e] << shift) | (uint32_t)lo);
        if (val > dmax)
            return ORC_BAD_FIELDS;
        v[e] = (uint16_t)val;
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* spec S1: blocks, groups and extents                                        */
/* ------------------------------------------------------------------------- */
static uint32_t rel_end(const uint32_t *g, int j)
{
    uint32_t word = g[1 + j / 2];
    return (j & 1) ? (word >> 16) : (word & 0xFFFFu);
}

uint64_t orc_encode_block(const void *counts, int w, int P, uint32_t *groups, uint8_t *payload)
{
    ensure_models();
    int G = (P + 31) / 32;
    uint64_t pos = 0;
    uint16_t v[512];
    uint8_t buf[2 + 1024];
    for (int g = 0; g < G; g++) {
        uint32_t *rec = groups + 17 * (size_t)g;
        memset(rec, 0, 17 * sizeof(uint32_t));
        rec[0] = (uint32_t)pos;
        uint32_t rel = 0;
        for (int j = 0; j < 32; j++) {
            int p = 32 * g + j;
            if (p < P) {
                for (int i = 0; i < 512; i++)
                    v[i] = (w == 2) ? ((const uint16_t *)counts)[(size_t)i * P + p]
                                    : ((const uint8_t *)counts)[(size_t)i * P + p];
                int len;
                orc_encode_stream(v, w, buf, &len);
                memcpy(payload + pos, buf, (size_t)len);
                pos += (uint64_t)len;
                rel += (uint32_t)len;
            }
            rec[1 + j / 2] |= (j & 1) ? (rel << 16) : rel;
        }
    }
    return pos;
}

/* extent of stream p of a block, with the offset checks of spec S7 */
static int extent(const uint32_t *groups, uint64_t len, int p, uint64_t *start, int *n)
{
    const uint32_t *g = groups + 17 * (size_t)(p / 32);
    int j = p % 32;
    uint32_t e1 = rel_end(g, j);
    uint32_t e0 = j ? rel_end(g, j - 1) : 0;
    if (e1 < e0)
        return ORC_BAD_OFFSETS;
    if ((uint64_t)g[0] + e1 > len)
        return ORC_BAD_OFFSETS;
    *start = (uint64_t)g[0] + e0;
    *n = (int)(e1 - e0);
    return ORC_OK;
}

int orc_block_masked_sum(const uint32_t *groups, const uint8_t *payload, uint64_t len,
                         int w, int P, const int32_t *pix, const int8_t *sign, int n,
                         int64_t out[512])
{
    uint16_t v[512];
    for (int k = 0; k < n; k++) {
        uint64_t st;
        int ln;
        int rc = extent(groups, len, pix[k], &st, &ln);
        if (rc)
            return rc;
        if (ln > 2 + 512 * w)
            return ORC_BAD_LENGTH;
        rc = orc_decode_stream(payload + st, ln, w, v);
        if (rc)
            return rc;
        for (int i = 0; i < 512; i++)
            out[i] += (int64_t)sign[k] * (int64_t)v[i];
    }
    (void)P;
    return ORC_OK;
}

int orc_decode_block(const uint32_t *groups, const uint8_t *payload, uint64_t len,
                     int w, int P, void *out)
{
    uint16_t v[512];
    for (int p = 0; p < P; p++) {
        uint64_t st;
        int ln;
        int rc = extent(groups, len, p, &st, &ln);
        if (rc)
            return rc;
        if (ln > 2 + 512 * w)
            return ORC_BAD_LENGTH;
        rc = orc_decode_stream(payload + st, ln, w, v);
        if (rc)
            return rc;
        for (int i = 0; i < 512; i++) {
            if (w == 2)
                ((uint16_t *)out)[(size_t)i * P + p] = v[i];
            else
                ((uint8_t *)out)[(size_t)i * P + p] = (uint8_t)v[i];
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* introspection for the tests                                                */
/* ------------------------------------------------------------------------- */
int orc_paired_size(const uint16_t v[512], int w, int model)
{
    ensure_models();
    uint8_t buf[2 + 2 + 64 * 12 + 332];
    int m;
    memset(buf, 0, sizeof(buf));
    return encode_paired(v, w, buf, model, &m);
}

void orc_stream_sizes(const uint16_t v[512], int w, int32_t info[4])
{
    ensure_models();
    uint8_t buf[2 + 2 + 64 * 12 + 332];
    int e, n = 0, m = -1;
    for (e = 0; e < 512; e++)
        n += v[e] != 0;
    memset(buf, 0, sizeof(buf));
    info[0] = n <= 256 ? 3 + (9 * n + 7) / 8 + n * w : 1 << 30;
    info[1] = encode_paired(v, w, buf, -1, &m);
    info[2] = 2 + 512 * w;
    info[3] = m;
}
