// kernels.cu -- sm_100a kernels of the paired-count resident.
//
// Page "Paired-count resident layout":
//  * "Operation pipeline" step 2 -- per-pixel 512-scan streams coded as count
//    pairs with 1024-state tANS from 32 Poisson pair models; empty, constant,
//    sparse and incompressible forms; grouped offsets (k_enc_streams,
//    k_enc_layout, k_enc_compact);
//  * step 4 -- a mask (or its difference from the previous mask) is turned
//    into a pixel list (k_plan) and the streams are decoded one thread per
//    stream with a 64-bit bit reservoir refilled four bytes at a time once per
//    three coded pairs, reduced warp-wide per 32 scans into exact integer
//    virtual images, optionally over every k-th block only (k_decode_reduce);
//  * step 3 -- the interaction index: exact per-scan sums of polar pixel
//    groups, built by one decode pass (k_index_sums, k_index_size,
//    k_index_pack); a full query takes the groups wholly inside its mask from
//    them and decodes the rest (k_plan_index, index items in k_decode_reduce);
//  * step 6 -- whole blocks decode back to native patterns (k_decode_blocks),
//    optionally with their float32 square-root amplitude (k_amplitude); any
//    scan range, a single frame included, decodes each stream only up to its
//    last needed pair (k_decode_range).
// Page "Backend Optimization Matrix", CUDA checkpoint rows: a dense mask as the
// cached full-detector image minus its complement (k_plan mode 2).
// Page "Backend Optimization Matrix", CoM/DPC rows: fused moment numerators
// and denominator over the same decode (k_moments).
// Bit-level choices follow the library's spec qem-pair-v2 (S1-S7).
//
// No kernel traps or asserts: malformed input sets flags in DevStatus and the
// affected lane contributes zeros.  Every loop ends: a fixed trip count, a
// position or counter that only advances, or a wait bounded by kWaitLimit
// polls that sets kErrWait when it runs out.
#include <cstdio>
#include <type_traits>

#include <map>
#include <mutex>
#include <utility>

#include "qem_internal.h"

namespace qem {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------
// Malformed-stream report (spec S7): a query only needs to know that some
// stream failed, so a flag is all that is kept (recording where would keep the
// block and pixel live through every decode loop).
__device__ __forceinline__ void report(DevStatus *st, uint32_t flag)
{
    atomicOr(&st->flags, flag);
}

// Shared-memory tables arrive by the bulk-copy engine: one thread starts the
// copies, which complete on an mbarrier; every thread waits on it before its
// first table read, so the copy overlaps the CTA's setup and its first stream
// opens.  The wait is bounded: past kWaitLimit polls it flags kErrWait and
// returns false (the query then reports an error instead of a result).
constexpr uint32_t kWaitLimit = 1u << 22;

__device__ __forceinline__ void tables_start(uint64_t *bar, uint32_t *s_dec, const uint32_t *dec_g,
                                             const uint32_t *runs_g, int skip_count)
{
    // one 4 KB table per model at its model's place: the run-event tables of
    // the models below skip_count, the decode tables of the others (two copies)
    const uint32_t b = static_cast<uint32_t>(__cvta_generic_to_shared(bar));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(b) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    const uint32_t run_bytes = static_cast<uint32_t>(skip_count) * kStates * 4u;
    const uint32_t dec_bytes = static_cast<uint32_t>(kModels - skip_count) * kStates * 4u;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(b), "r"(run_bytes + dec_bytes)
                 : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(s_dec + skip_count * kStates))),
                 "l"(dec_g + skip_count * kStates), "r"(dec_bytes), "r"(b)
                 : "memory");
    if (run_bytes)
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                         static_cast<uint32_t>(__cvta_generic_to_shared(s_dec))),
                     "l"(runs_g), "r"(run_bytes), "r"(b)
                     : "memory");
}

__device__ __forceinline__ bool tables_wait(uint64_t *bar, DevStatus *st)
{
    const uint32_t b = static_cast<uint32_t>(__cvta_generic_to_shared(bar));
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
        uint32_t done;
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(done)
                     : "r"(b)
                     : "memory");
        if (done)
            return true;
    }
    atomicOr(&st->flags, kErrWait);
    return false;
}

// Forward LSB-first bit reader over aligned 32-bit little-endian words: a
// 64-bit reservoir (lo, hi) holding `n` valid bits.  Words are addressed by
// index from `first` (the aligned word holding the stream's first byte), and
// loads never pass word `li` (the aligned word at or after the stream's end),
// so a malformed stream reads repeated bytes inside its arena instead of
// running off the end; the caller's length checks then reject it.
struct Bits {
    const uint32_t *first;
    uint32_t wi;     // index of the next word to enter the reservoir
    uint32_t li;     // last word that may be loaded
    uint32_t nx0;    // words wi and wi + 1, loaded two top-ups ahead
    uint32_t nx1;
    uint32_t lo, hi;
    int n;
    int lead;        // bits of the first word before the stream start

    __device__ __forceinline__ void init(const uint8_t *p, const uint8_t *end)
    {
        const uintptr_t a = reinterpret_cast<uintptr_t>(p);
        const uintptr_t f = a & ~static_cast<uintptr_t>(3);
        first = reinterpret_cast<const uint32_t *>(f);
        li = static_cast<uint32_t>((((reinterpret_cast<uintptr_t>(end) + 3) & ~static_cast<uintptr_t>(3)) - f) >> 2);
        lead = static_cast<int>(a & 3) * 8;
        lo = __ldg(first) >> lead;
        hi = 0u;
        n = 32 - lead;
        wi = 1u;
        nx0 = __ldg(first + min(1u, li));
        nx1 = __ldg(first + min(2u, li));
    }
    // requires n < 32; the word it adds was loaded two top-ups earlier, and
    // the load for the one after next is issued here
    __device__ __forceinline__ void refill()
    {
        const uint32_t w = nx0;
        nx0 = nx1;
        nx1 = __ldg(first + min(wi + 2u, li));
        lo |= w << n;
        hi |= __funnelshift_l(w, 0u, n);
        n += 32;
        ++wi;
    }
    // nb < 32 and nb <= n
    __device__ __forceinline__ uint32_t get(int nb)
    {
        const uint32_t v = lo & ((1u << nb) - 1u);
        lo = __funnelshift_r(lo, hi, nb);
        hi >>= nb;
        n -= nb;
        return v;
    }
    // bits consumed since init
    __device__ __forceinline__ long long consumed() const
    {
        return 32ll * wi - lead - n;
    }
};

__device__ __forceinline__ uint32_t load_native(const uint8_t *p, int w)
{
    return w == 2 ? static_cast<uint32_t>(__ldg(p)) | (static_cast<uint32_t>(__ldg(p + 1)) << 8)
                  : static_cast<uint32_t>(__ldg(p));
}

// Parsed stream (spec S2/S3) with its readers.
struct Stream {
    int form;            // Form, kEmpty also for inactive or rejected lanes
    int model;
    int shift;
    uint32_t base;
    uint32_t c;          // constant value / sparse count
    uint32_t x;          // tANS state minus 1024 (state A: every pair, or the even pairs)
    uint32_t x2;         // state B minus 1024 (odd pairs) when two
    bool two;            // paired stream coded with two interleaved states (spec S3/S5)
    const uint8_t *s;
    uint32_t len;
    uint32_t tans_len;   // paired: bytes of the tANS section
    Bits bt;             // paired: tANS section; literal: values; sparse: positions
    Bits br;             // paired: raw section; sparse: values
};

// Locate stream (b, p) through its group record and check the offsets (S1, S7).
__device__ __forceinline__ bool locate(const View &v, long long b, int p, const uint8_t *&s,
                                       uint32_t &len, DevStatus *st)
{
    const uint32_t *rec = v.groups + (static_cast<long long>(b) * v.G + (p >> 5)) * kGroupWords;
    const int j = p & 31;
    const uint32_t base = __ldg(rec);
    const uint32_t w1 = __ldg(rec + 1 + (j >> 1));
    const uint32_t e1 = (j & 1) ? (w1 >> 16) : (w1 & 0xFFFFu);
    uint32_t e0 = 0;
    if (j) {
        const uint32_t w0 = __ldg(rec + 1 + ((j - 1) >> 1));
        e0 = ((j - 1) & 1) ? (w0 >> 16) : (w0 & 0xFFFFu);
    }
    const uint32_t blen = __ldg(v.blk_len + b);
    if (e1 < e0 || static_cast<uint64_t>(base) + e1 > blen) {
        report(st, kErrOffsets);
        return false;
    }
    s = reinterpret_cast<const uint8_t *>(__ldg(v.blk_ptr + b)) + base + e0;
    len = e1 - e0;
    return true;
}

// Ask L2 for every 128-byte line of a stream up front: the decoder then
// reads it word by word along a dependent chain, and each of those reads
// would otherwise wait for HBM.  Prefetches take no registers and never fault.
__device__ __forceinline__ void prefetch_stream(const uint8_t *s, uint32_t len)
{
    // lines after the one holding the header (that one is being read already)
    const uintptr_t a = (reinterpret_cast<uintptr_t>(s) & ~static_cast<uintptr_t>(127)) + 128;
    const uintptr_t e = reinterpret_cast<uintptr_t>(s) + len;
    for (uintptr_t q = a; q < e; q += 128)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(q));
}

// Parse the header and set the readers up; false (after reporting) if malformed.
__device__ bool open_stream(Stream &S, int w, DevStatus *st)
{
    if (S.len == 0) {
        S.form = kEmpty;
        return true;
    }
    prefetch_stream(S.s, S.len);
    if (S.len < 2) {
        report(st, kErrLength);
        return false;
    }
    const uint32_t hdr = static_cast<uint32_t>(__ldg(S.s)) | (static_cast<uint32_t>(__ldg(S.s + 1)) << 8);
    if (hdr >> 13) {
        report(st, kErrReserved);
        return false;
    }
    S.form = static_cast<int>(hdr & 7);
    S.model = static_cast<int>((hdr >> 3) & 31);
    S.shift = static_cast<int>((hdr >> 8) & 15);
    const int has_base = static_cast<int>((hdr >> 12) & 1);
    if (S.form < kConstant || S.form > kLiteral) {
        report(st, kErrForm);
        return false;
    }
    if (S.form != kPaired && (S.model | S.shift | has_base)) {
        report(st, kErrFields);
        return false;
    }
    const uint8_t *end = S.s + S.len;
    if (S.form == kConstant) {
        if (S.len != static_cast<uint32_t>(2 + w)) {
            report(st, kErrLength);
            return false;
        }
        S.c = load_native(S.s + 2, w);
        if (S.c == 0) {
            report(st, kErrConstant);
            return false;
        }
        return true;
    }
    if (S.form == kLiteral) {
        if (S.len != static_cast<uint32_t>(2 + 512 * w)) {
            report(st, kErrLength);
            return false;
        }
        S.bt.init(S.s + 2, end);
        return true;
    }
    if (S.form == kSparse) {
        if (S.len < 3) {
            report(st, kErrLength);
            return false;
        }
        S.c = static_cast<uint32_t>(__ldg(S.s + 2)) + 1u;
        const uint32_t pbytes = (9u * S.c + 7u) / 8u;
        if (S.len != 3u + pbytes + S.c * static_cast<uint32_t>(w)) {
            report(st, kErrLength);
            return false;
        }
        S.bt.init(S.s + 3, end);
        S.br.init(S.s + 3 + pbytes, end);
        return true;
    }
    // paired
    if (S.shift > 8 * w - 4) {
        report(st, kErrFields);
        return false;
    }
    uint32_t off = 2;
    S.base = 0;
    if (has_base) {
        if (S.len < off + static_cast<uint32_t>(w)) {
            report(st, kErrLength);
            return false;
        }
        S.base = load_native(S.s + off, w);
        off += static_cast<uint32_t>(w);
    }
    const uint32_t raw_off = off;
    off += 64u * static_cast<uint32_t>(S.shift);
    if (S.len < off + 2u) {
        report(st, kErrLength);
        return false;
    }
    S.tans_len = S.len - off;
    S.br.init(S.s + raw_off, end);
    S.bt.init(S.s + off, end);
    if (S.bt.n < 10)
        S.bt.refill();
    S.x = S.bt.get(10);
    S.two = S.model >= kOneStateModels;
    S.x2 = 0;
    if (S.two) {
        if (S.bt.n < 10)
            S.bt.refill();
        S.x2 = S.bt.get(10);
    }
    return true;
}

// End-of-stream checks of a paired stream (S5/S7): final state 1024, section
// length exactly ceil(T/8), zero pad bits.
__device__ bool close_paired(Stream &S, DevStatus *st)
{
    if (S.x != 0 || S.x2 != 0) {
        report(st, kErrState);
        return false;
    }
    const long long T = S.bt.consumed();
    if ((T + 7) / 8 != static_cast<long long>(S.tans_len)) {
        report(st, kErrLength);
        return false;
    }
    const int pad = static_cast<int>(8ll * S.tans_len - T);
    if (pad) {
        if (S.bt.n < pad)
            S.bt.refill();
        if (S.bt.get(pad) != 0u) {
            report(st, kErrPad);
            return false;
        }
    }
    return true;
}

// One tANS decode step with no raw bits: returns the table entry.
__device__ __forceinline__ uint32_t tans_step(Stream &S, const uint32_t *dec)
{
    const uint32_t ent = dec[S.x];
    const int nb = static_cast<int>((ent >> 10) & 15u);
    S.x = (ent & 1023u) | S.bt.get(nb);      // newbase's low nb bits are zero
    return ent;
}

// The u8 fast path (paired, no base, no raw bits): one tANS step written out
// so that the state update, the bit consumption and the packed pair
// (hi_a | hi_b << 16) cost as few integer-pipe instructions as possible: the
// table address is formed by mad (FMA pipe), the mask by bmsk, the new state
// by one lop3 (newbase | (bits & mask); newbase's low nb bits are zero), the
// reservoir shift by a funnel shift, the pair by prmt.
// The same step in two halves, for two interleaved states: the table load
// (which depends only on the state) and the bit consumption (which depends on
// the reservoir, so state B's consumption follows state A's), so that both
// states' loads are in flight together.
// tab_load as a volatile statement: it keeps its place before the shared
// reductions that follow it in the run-event loop
__device__ __forceinline__ uint32_t tab_load_ordered(uint32_t x, uint32_t dec_sa)
{
    uint32_t e;
    asm volatile("{\n\t"
                 ".reg .b32 a;\n\t"
                 "mad.lo.u32 a, %1, 4, %2;\n\t"
                 "ld.shared.u32 %0, [a];\n\t"
                 "}"
                 : "=r"(e)
                 : "r"(x), "r"(dec_sa));
    return e;
}

__device__ __forceinline__ uint32_t tab_load(uint32_t x, uint32_t dec_sa)
{
    uint32_t e;
    asm("{\n\t"
        ".reg .b32 a;\n\t"
        "mad.lo.u32 a, %1, 4, %2;\n\t"
        "ld.shared.u32 %0, [a];\n\t"
        "}"
        : "=r"(e)
        : "r"(x), "r"(dec_sa));
    return e;
}

__device__ __forceinline__ uint32_t consume(uint32_t e, uint32_t &x, uint32_t &lo, uint32_t &hi, int &n)
{
    uint32_t pk, nb;
    asm("{\n\t"
        ".reg .b32 m, t;\n\t"
        "bfe.u32 %1, %6, 10, 4;\n\t"
        "bmsk.clamp.b32 m, 0, %1;\n\t"
        "and.b32 t, %4, m;\n\t"
        "lop3.b32 %3, %6, 1023, t, 0xEA;\n\t"
        "shf.r.clamp.b32 %4, %4, %5, %1;\n\t"
        "shr.b32 %5, %5, %1;\n\t"
        "prmt.b32 %0, %6, 0, 0x4342;\n\t"
        "}"
        : "=r"(pk), "=r"(nb), "+r"(n), "+r"(x), "+r"(lo), "+r"(hi)
        : "r"(e));
    n -= static_cast<int>(nb);
    return pk;
}

// Decode 16 pairs (32 scans) of a paired stream into values v[32] (general
// path: base and raw low bits).  Refill policy: the tANS reservoir is topped up
// before pairs 0, 3, 6, 9, 12, 15 of the segment (<= 30 bits per 3 pairs);
// the raw reservoir whenever it holds fewer than 2*shift bits.
__device__ __forceinline__ void paired_segment(Stream &S, const uint32_t *dec, uint32_t (&v)[32],
                                               uint32_t &over)
{
    const uint32_t mask = (1u << S.shift) - 1u;
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) {
        if (jj % 3 == 0 && S.bt.n < 30)
            S.bt.refill();
        if (S.br.n < 2 * S.shift)
            S.br.refill();
        // a segment starts at an even pair: odd jj is an odd pair, on state B
        // when the stream has two states
        uint32_t ent;
        if ((jj & 1) && S.two) {
            ent = dec[S.x2];
            S.x2 = (ent & 1023u) | S.bt.get(static_cast<int>((ent >> 10) & 15u));
        } else {
            ent = tans_step(S, dec);
        }
        const uint32_t lo = S.br.get(2 * S.shift);
        const uint32_t va = S.base + ((((ent >> 16) & 0xFFu) << S.shift) | (lo & mask));
        const uint32_t vb = S.base + (((ent >> 24) << S.shift) | ((lo >> S.shift) & mask));
        over |= va | vb;
        v[2 * jj] = va;
        v[2 * jj + 1] = vb;
    }
}

// ---------------------------------------------------------------------------
// synthetic generator (a1, bench/test input only)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void k_generate(T *__restrict__ out, uint64_t seed, int64_t scan0, int64_t n_scans, int P,
                           const uint32_t *__restrict__ pclass, const uint4 *__restrict__ desc,
                           const uint64_t *__restrict__ thr, uint32_t dmax)
{
    for (int64_t s = blockIdx.y; s < n_scans; s += gridDim.y) {
        for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < P; p += gridDim.x * blockDim.x) {
            const uint64_t idx = static_cast<uint64_t>(scan0 + s) * static_cast<uint64_t>(P) +
                                 static_cast<uint64_t>(p) + 1ull;
            uint64_t z = seed + idx * 0x9E3779B97F4A7C15ull;
            z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
            z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
            z = z ^ (z >> 31);
            const uint4 d = desc[pclass[p]];
            uint32_t val;
            if (d.x == 0u) {
                const uint64_t u = z >> 11;
                const uint64_t *t = thr + d.y;
                int lo = 0, hi = static_cast<int>(d.z) - 1;
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (u >= __ldg(t + mid))
                        lo = mid + 1;
                    else
                        hi = mid;
                }
                val = static_cast<uint32_t>(lo < 0 ? 0 : lo);
            } else if (d.x == 1u) {
                val = static_cast<uint32_t>(z) & dmax;
            } else {
                val = d.w;
            }
            out[s * P + p] = static_cast<T>(val < dmax ? val : dmax);
        }
    }
}

// ---------------------------------------------------------------------------
// encoder (a2-a4)
// ---------------------------------------------------------------------------
// Counts of scans i0 .. i0 + N - 1 of one pixel column (stride P): the loads
// are issued together, so a thread that reads a stream's counts waits for one
// round trip per batch rather than one per scan.
constexpr int kColBatch = 16;

template <typename T, int N>
__device__ __forceinline__ void load_column(const T *col, int P, int i0, uint32_t (&x)[N])
{
#pragma unroll
    for (int u = 0; u < N; ++u)
        x[u] = static_cast<uint32_t>(__ldg(col + static_cast<size_t>(i0 + u) * P));
}

constexpr int kEncThreads = 256;

// a2+a3: per stream (one thread): statistics, base/shift, hi histogram, model
// selection (spec S6), backward tANS pass writing the section into this
// stream's scratch slot from the top down (so the decoder reads it forward),
// and the form decision.  desc: x = length, y = header | T << 16,
// z = base (or constant value) | nnz << 16, w = offset (filled by layout).
template <typename T>
__global__ void __launch_bounds__(kEncThreads, 6) k_enc_streams(const T *__restrict__ counts, int P, int nblk,
                                                            Tables tb, uint4 *__restrict__ desc,
                                                            uint32_t *__restrict__ slots,
                                                            unsigned long long *__restrict__ stats,
                                                            uint8_t *__restrict__ pclass)
{
    constexpr uint32_t W = sizeof(T);
    __shared__ uint32_t s_cost[kModels * 16];
    __shared__ uint32_t s_amax[kModels];
    __shared__ uint16_t s_hist[16][kEncThreads];
    __shared__ unsigned int s_stats[5 + kModels];
    const int tid = threadIdx.x;
    for (int i = tid; i < kModels * 16; i += kEncThreads)
        s_cost[i] = tb.cost[i];
    if (tid < kModels)
        s_amax[tid] = tb.amax[tid];
    if (tid < 5 + kModels)
        s_stats[tid] = 0;
    __syncthreads();

    const long long sid = static_cast<long long>(blockIdx.x) * kEncThreads + tid;
    if (sid < static_cast<long long>(nblk) * P) {
        const int b = static_cast<int>(sid / P);
        const int p = static_cast<int>(sid - static_cast<long long>(b) * P);
        const T *col = counts + static_cast<size_t>(b) * kScans * P + p;

        uint32_t nnz = 0, mn = 0xFFFFFFFFu, mx = 0;
        uint32_t c0 = 0, c1 = 0, c2 = 0, c3 = 0;      // first four nonzeros: scan | value << 16
        // the histogram of the counts below 16 is taken in the same pass: when no
        // count reaches 16 it is the hi histogram after the base (no shift).  Only
        // nonzero counts do any work here (most counts of a low-dose pixel are
        // 0): the zeros' bin, the minimum and the statistics follow from nnz.
#pragma unroll
        for (int v = 1; v < 16; ++v)
            s_hist[v][tid] = 0;
        constexpr int kB = 8;           // loads in flight per thread (occupancy bounds the batch)
        for (int i0 = 0; i0 < kScans; i0 += kB) {
            uint32_t x[kB];
            load_column(col, P, i0, x);
#pragma unroll
            for (int u = 0; u < kB; ++u) {
                const uint32_t v = x[u];
                if (v) {
                    if (v < 16u)
                        s_hist[v][tid] += 1;
                    if (nnz < 4u) {
                        const uint32_t e = static_cast<uint32_t>(i0 + u) | (v << 16);
                        c0 = nnz == 0u ? e : c0;
                        c1 = nnz == 1u ? e : c1;
                        c2 = nnz == 2u ? e : c2;
                        c3 = nnz == 3u ? e : c3;
                    }
                    ++nnz;
                    mn = min(mn, v);
                    mx = max(mx, v);
                }
            }
        }
        s_hist[0][tid] = static_cast<uint16_t>(kScans - nnz);
        if (nnz < static_cast<uint32_t>(kScans))
            mn = 0u;
        uint4 d = make_uint4(0u, 0u, 0u, 0u);
        int form = kEmpty, model = -1;
        if (nnz == 0u) {
            form = kEmpty;
        } else if (mn == mx) {
            form = kConstant;
            d.x = 2u + W;
            d.y = kConstant;
            d.z = mn;
        } else {
            const uint32_t lit = 2u + 512u * W;
            const uint32_t sparse = nnz <= 256u ? 3u + (9u * nnz + 7u) / 8u + nnz * W : 0xFFFFFFFFu;
            const uint32_t has_base = mn > 0u ? 1u : 0u;
            const uint32_t base = has_base ? mn : 0u;
            const int span_bits = 32 - __clz(static_cast<int>(mx - base));
            const int shift = span_bits > 4 ? span_bits - 4 : 0;

            const bool small = mx < 16u;             // every hi = count - base
            if (!small) {
#pragma unroll
                for (int v = 0; v < 16; ++v)
                    s_hist[v][tid] = 0;
                const T *q = col;
#pragma unroll 8
                for (int i = 0; i < kScans; ++i, q += P)
                    s_hist[(static_cast<uint32_t>(*q) - base) >> shift][tid] += 1;
            }
            const uint32_t maxhi = (mx - base) >> shift;
            const uint32_t hoff = small ? base : 0u;
            uint32_t h[16];
#pragma unroll
            for (int v = 0; v < 16; ++v)
                h[v] = v + hoff < 16u ? s_hist[v + hoff][tid] : 0u;
            uint32_t best = 0xFFFFFFFFu;
            model = kModels - 1;
            for (int m = 0; m < kModels; ++m) {
                if (s_amax[m] < maxhi)
                    continue;
                uint32_t c = 0;
#pragma unroll
                for (int v = 0; v < 16; ++v)
                    c += h[v] * s_cost[m * 16 + v];
                if (c < best) {
                    best = c;
                    model = m;
                }
            }

            // backward tANS pass, chunks prepended at the low end of `acc`
            const uint32_t *esym = tb.enc_sym + model * 256;
            const uint16_t *eslot = tb.enc_slot + model * kStates;
            uint32_t *slot = slots + static_cast<size_t>(sid) * kSlotWords;
            int wi = kSlotWords - 1;
            uint64_t acc = 0;
            int nacc = 0;
            // models 8-31 code pair j on state A (even j) or B (odd j); both start
            // at 1024 after pair 255 (spec S3/S5)
            const bool two = model >= kOneStateModels;
            uint32_t Tbits = two ? 20u : 10u;
            uint32_t XA = kStates, XB = kStates;
            auto push = [&](uint32_t bits, uint32_t k) {
                acc = (acc << k) | bits;
                nacc += static_cast<int>(k);
                if (nacc >= 32) {
                    slot[wi--] = static_cast<uint32_t>(acc >> (nacc - 32));
                    nacc -= 32;
                }
            };
            // one tANS encode step of pair (ca, cb) from state X: the bits to emit
            // (chunk, k) and the new state
            auto step = [&](uint32_t ca, uint32_t cb, uint32_t &X, uint32_t &k) {
                const uint32_t a = (ca - base) >> shift;
                const uint32_t bb = (cb - base) >> shift;
                const uint32_t es = __ldg(esym + a + 16u * bb);
                const uint32_t f = es & 0x7FFu;
                const uint32_t cum = (es >> 11) & 0x7FFu;
                const uint32_t k0 = es >> 22;
                k = k0 - ((X >> k0) < f ? 1u : 0u);
                const uint32_t chunk = X & ((1u << k) - 1u);
                const uint32_t y = X >> k;
                X = kStates + __ldg(eslot + cum + (y - f));
                return chunk;
            };
            // the counts are read again kEB scans at a time, from the top (the
            // loads of a batch are issued together)
            constexpr int kEB = 8;
            if (__all_sync(__activemask(), two)) {
                // every stream of these lanes has two states: odd pair j on B and
                // even pair j - 1 on A are independent steps
                for (int i0 = kScans - kEB; i0 >= 0; i0 -= kEB) {
                    uint32_t x[kEB];
                    load_column(col, P, i0, x);
#pragma unroll
                    for (int u = kEB / 2 - 1; u > 0; u -= 2) {
                        uint32_t kb, ka;
                        const uint32_t cb = step(x[2 * u], x[2 * u + 1], XB, kb);
                        const uint32_t ca = step(x[2 * u - 2], x[2 * u - 1], XA, ka);
                        push(cb, kb);
                        push(ca, ka);
                        Tbits += kb + ka;
                    }
                }
            } else {
                for (int i0 = kScans - kEB; i0 >= 0; i0 -= kEB) {
                    uint32_t x[kEB];
                    load_column(col, P, i0, x);
#pragma unroll
                    for (int u = kEB / 2 - 1; u >= 0; --u) {
                        const bool on_b = two && (u & 1);     // pair i0 / 2 + u; i0 / 2 is even
                        uint32_t X = on_b ? XB : XA;
                        uint32_t k;
                        const uint32_t chunk = step(x[2 * u], x[2 * u + 1], X, k);
                        if (on_b)
                            XB = X;
                        else
                            XA = X;
                        push(chunk, k);
                        Tbits += k;
                    }
                }
            }
            // the section starts with x_A, then x_B: prepended last, in reverse
            if (two)
                push(XB - kStates, 10u);
            push(XA - kStates, 10u);
            if (nacc > 0)
                slot[wi] = static_cast<uint32_t>(acc << (32 - nacc));
            {
                // move the section (bits [32*kSlotWords - T, 32*kSlotWords) of the
                // slot) down to bit 0, zero-filled above its end, so that the
                // compaction copies plain bytes
                const int o0 = 32 * kSlotWords - static_cast<int>(Tbits);
                const int w0 = o0 >> 5, sh = o0 & 31;
                const int nw = static_cast<int>((Tbits + 31u) >> 5);
                for (int i = 0; i < nw; ++i) {
                    const uint32_t a = slot[w0 + i];
                    const uint32_t c = w0 + i + 1 < kSlotWords ? slot[w0 + i + 1] : 0u;
                    slot[i] = __funnelshift_r(a, c, sh);
                }
            }

            const uint32_t paired = 2u + has_base * W + 64u * static_cast<uint32_t>(shift) + (Tbits + 7u) / 8u;
            uint32_t size;
            if (sparse <= paired + 1u) {
                form = kSparse;
                size = sparse;
            } else {
                form = kPaired;
                size = paired;
            }
            if (size >= lit) {
                form = kLiteral;
                size = lit;
            }
            d.x = size;
            if (form == kPaired)
                d.y = static_cast<uint32_t>(kPaired) | (static_cast<uint32_t>(model) << 3) |
                      (static_cast<uint32_t>(shift) << 8) | (has_base << 12) | (Tbits << 16);
            else
                d.y = static_cast<uint32_t>(form);
            d.z = base | (nnz << 16);
            if (form == kSparse && size - 2u <= static_cast<uint32_t>(kSlotWords) * 4u) {
                // the column is hot in L1 now: write the sparse payload (n-1,
                // 9-bit positions, values) into the slot for the compaction to copy
                uint8_t *o = reinterpret_cast<uint8_t *>(slot);
                uint32_t k = 0, acc = 0;
                int nacc = 0;
                o[k++] = static_cast<uint8_t>(nnz - 1u);
                auto put_pos = [&](uint32_t i) {
                    acc |= i << nacc;
                    nacc += 9;
                    while (nacc >= 8) {
                        o[k++] = static_cast<uint8_t>(acc & 0xFFu);
                        acc >>= 8;
                        nacc -= 8;
                    }
                };
                auto put_val = [&](uint32_t v) {
                    o[k++] = static_cast<uint8_t>(v & 0xFFu);
                    if (W == 2)
                        o[k++] = static_cast<uint8_t>(v >> 8);
                };
                if (nnz <= 4u) {
                    // the first pass kept them: no further reads
                    const uint32_t c[4] = {c0, c1, c2, c3};
                    for (uint32_t j = 0; j < nnz; ++j)
                        put_pos(c[j] & 0xFFFFu);
                    if (nacc > 0)
                        o[k++] = static_cast<uint8_t>(acc & 0xFFu);
                    for (uint32_t j = 0; j < nnz; ++j)
                        put_val(c[j] >> 16);
                } else {
                    const T *q = col;
                    for (int i = 0; i < kScans; ++i, q += P)
                        if (*q)
                            put_pos(static_cast<uint32_t>(i));
                    if (nacc > 0)
                        o[k++] = static_cast<uint8_t>(acc & 0xFFu);
                    q = col;
                    for (int i = 0; i < kScans; ++i, q += P)
                        if (*q)
                            put_val(*q);
                }
                d.y |= 1u << 16;          // the payload after the header is in the slot
            }
        }
        desc[sid] = d;
        if (pclass && b == 0) {
            // the pixel's cost class, from its block-0 stream: 1 = light (empty,
            // sparse, or paired decoded by runs), 0 = heavy (decoded pair by pair)
            const uint32_t hdr = d.y & 0xFFFFu;
            const bool runs = form == kPaired && ((hdr >> 8) & 0x1Fu) == 0u &&
                              ((tb.skip_models >> model) & 1u);
            pclass[p] = (form == kEmpty || form == kSparse || runs) ? 1 : 0;
        }
        atomicAdd(&s_stats[form], 1u);
        if (form == kPaired)
            atomicAdd(&s_stats[5 + model], 1u);
    }
    __syncthreads();
    if (tid < 5 + kModels && s_stats[tid])
        atomicAdd(stats + tid, static_cast<unsigned long long>(s_stats[tid]));
}

constexpr int kLayoutThreads = 1024;

__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t x, uint32_t *s_warp, uint32_t &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(kFull, inc, o);
        if (lane >= o)
            inc += y;
    }
    if (lane == 31)
        s_warp[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        uint32_t v = lane < nw ? s_warp[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(kFull, v, o);
            if (lane >= o)
                v += y;
        }
        if (lane < nw)
            s_warp[lane] = v;          // inclusive warp prefix
    }
    __syncthreads();
    total = s_warp[(blockDim.x >> 5) - 1];
    const uint32_t before = warp ? s_warp[warp - 1] : 0u;
    return before + inc - x;
}

// a4 (first half): per block, exclusive scan of stream lengths in pixel order
// -> per-stream offsets (desc.w), block length, and the group records (S1).
// Each warp scans one contiguous chunk of pixels 32 at a time (coalesced
// descriptor reads and writes); a block-wide scan joins the chunks; then
// each warp writes whole group records (lane j holds stream j's end).
__global__ void __launch_bounds__(kLayoutThreads) k_enc_layout(uint4 *__restrict__ desc, int P, int G,
                                                              uint32_t *__restrict__ groups,
                                                              uint32_t *__restrict__ blk_len)
{
    __shared__ uint32_t s_warp[32];
    const int b = blockIdx.x;
    uint4 *d = desc + static_cast<size_t>(b) * P;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int NW = kLayoutThreads / 32;
    const int chunk = ((P + NW - 1) / NW + 31) & ~31;
    const int c0 = min(P, warp * chunk), c1 = min(P, c0 + chunk);
    uint32_t local = 0;
    for (int p = c0 + lane; p < c1; p += 32)
        local += d[p].x;
#pragma unroll
    for (int o = 16; o; o >>= 1)
        local += __shfl_xor_sync(kFull, local, o);
    uint32_t total;
    const uint32_t mine = lane == 0 ? local : 0u;
    uint32_t run = __shfl_sync(kFull, block_exclusive_scan(mine, s_warp, total), 0);
    for (int base = c0; base < c1; base += 32) {
        const int p = base + lane;
        const uint32_t len = p < c1 ? d[p].x : 0u;
        uint32_t inc = len;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(kFull, inc, o);
            if (lane >= o)
                inc += y;
        }
        if (p < c1)
            d[p].w = run + inc - len;
        run += __shfl_sync(kFull, inc, 31);
    }
    if (threadIdx.x == 0)
        blk_len[b] = total;
    __syncthreads();
    uint32_t *gb = groups + static_cast<size_t>(b) * G * kGroupWords;
    for (int g = warp; g < G; g += NW) {
        const int p = 32 * g + lane;
        const uint32_t base = d[32 * g].w;
        // the last real stream's end repeats over the padding lanes of the last group
        const int q = min(p, P - 1);
        const uint4 dq = d[q];
        const uint32_t end = dq.w + dq.x - base;
        const uint32_t other = __shfl_down_sync(kFull, end, 1);
        uint32_t *rec = gb + static_cast<size_t>(g) * kGroupWords;
        if (lane == 0)
            rec[0] = base;
        if ((lane & 1) == 0)
            rec[1 + lane / 2] = end | (other << 16);
    }
}

// Write one stream's bytes (header and form payload, spec S2/S3) at o, except
// the section the encoder staged in the stream's slot (the tANS section of a
// paired stream, the payload of a sparse stream that was staged whole).  The
// section's place in the stream (byte offset) and length are returned in
// sec_at and sec_len (0 when there is none).
template <typename T>
__device__ __forceinline__ void write_head(uint8_t *o, const T *col, int P, const uint4 d, uint32_t &sec_at,
                                           uint32_t &sec_len)
{
    constexpr uint32_t W = sizeof(T);
    const uint32_t hdr = d.y & 0xFFFFu;     // (bits 16+ of d.y: T for paired, a flag for sparse)
    const int form = static_cast<int>(hdr & 7u);
    o[0] = static_cast<uint8_t>(hdr & 0xFFu);
    o[1] = static_cast<uint8_t>(hdr >> 8);
    uint32_t k = 2;
    sec_at = 0;
    sec_len = 0;
    auto put = [&](uint32_t v) {
        o[k++] = static_cast<uint8_t>(v & 0xFFu);
        if (W == 2)
            o[k++] = static_cast<uint8_t>(v >> 8);
    };
    if (form == kConstant) {
        put(d.z & 0xFFFFu);
    } else if (form == kLiteral) {
        for (int i0 = 0; i0 < kScans; i0 += kColBatch) {
            uint32_t x[kColBatch];
            load_column(col, P, i0, x);
#pragma unroll
            for (int u = 0; u < kColBatch; ++u)
                put(x[u]);
        }
    } else if (form == kSparse && ((d.y >> 16) & 1u)) {
        sec_at = k;
        sec_len = d.x - 2u;
    } else if (form == kSparse) {
        const uint32_t nnz = d.z >> 16;
        o[k++] = static_cast<uint8_t>(nnz - 1u);
        uint32_t acc = 0;
        int nacc = 0;
        for (int i0 = 0; i0 < kScans; i0 += kColBatch) {
            uint32_t x[kColBatch];
            load_column(col, P, i0, x);
#pragma unroll
            for (int u = 0; u < kColBatch; ++u) {
                if (x[u]) {
                    acc |= static_cast<uint32_t>(i0 + u) << nacc;
                    nacc += 9;
                    while (nacc >= 8) {
                        o[k++] = static_cast<uint8_t>(acc & 0xFFu);
                        acc >>= 8;
                        nacc -= 8;
                    }
                }
            }
        }
        if (nacc > 0)
            o[k++] = static_cast<uint8_t>(acc & 0xFFu);
        for (int i0 = 0; i0 < kScans; i0 += kColBatch) {
            uint32_t x[kColBatch];
            load_column(col, P, i0, x);
#pragma unroll
            for (int u = 0; u < kColBatch; ++u)
                if (x[u])
                    put(x[u]);
        }
    } else {
        const int shift = static_cast<int>((hdr >> 8) & 15u);
        const uint32_t base = d.z & 0xFFFFu;
        if ((hdr >> 12) & 1u)
            put(base);
        if (shift) {
            const uint32_t mask = (1u << shift) - 1u;
            uint32_t acc = 0;
            int nacc = 0;
            for (int i0 = 0; i0 < kScans; i0 += kColBatch) {
                uint32_t x[kColBatch];
                load_column(col, P, i0, x);
#pragma unroll
                for (int u = 0; u < kColBatch; ++u) {
                    acc |= ((x[u] - base) & mask) << nacc;
                    nacc += shift;
                    while (nacc >= 8) {
                        o[k++] = static_cast<uint8_t>(acc & 0xFFu);
                        acc >>= 8;
                        nacc -= 8;
                    }
                }
            }
        }
        // the tANS section starts at byte 0 of the stream's 16-byte aligned slot
        sec_at = k;
        sec_len = ((d.y >> 16) + 7u) / 8u;
    }
}

constexpr int kCompactThreads = 128;
constexpr int kCompactBytes = 32 * 1024;   // staged byte range per CTA (dynamic shared memory)
constexpr int kCompactUnroll = 4;          // slot loads a thread has in flight

// a4 (second half): write every stream's bytes at blk_dst[b] + offset.  A CTA
// takes 128 consecutive pixels of one block, whose streams are contiguous in
// the payload.  When their byte range fits, it is assembled in shared memory
// (placed congruent to the destination modulo 16) and stored with aligned
// 16-byte writes, bytes only at the two ragged ends:
//   1. the range is zeroed;
//   2. each thread writes its stream's own bytes (header, base, raw low bits,
//      the forms built from the counts);
//   3. the staged sections of all the CTA's streams are cut into 16-byte
//      chunks of their slots, numbered across the CTA by a scan, and every
//      thread takes chunks in turn, kCompactUnroll loads in flight before it
//      ORs each chunk into place as five shifted words (the bytes around it
//      belong to other streams or are still zero).
// A larger range (incompressible data) is written in place, one stream per
// thread.
template <typename T>
__global__ void __launch_bounds__(kCompactThreads) k_enc_compact(const T *__restrict__ counts, int P, int nblk,
                                                                const uint4 *__restrict__ desc,
                                                                const uint32_t *__restrict__ slots,
                                                                const unsigned long long *__restrict__ blk_dst)
{
    extern __shared__ __align__(16) uint8_t s_buf[];     // kCompactBytes + 32
    __shared__ uint32_t s_warp[32];
    __shared__ uint32_t s_chunk0[kCompactThreads];       // first chunk number of each stream's section
    __shared__ uint32_t s_at[kCompactThreads];           // section start in s_buf
    __shared__ uint32_t s_len[kCompactThreads];          // section bytes
    const int b = blockIdx.y;
    const int p0 = blockIdx.x * kCompactThreads;
    const int p1 = min(P, p0 + kCompactThreads);
    const int p = p0 + static_cast<int>(threadIdx.x);
    const long long sid = static_cast<long long>(b) * P + p;
    uint8_t *blk = reinterpret_cast<uint8_t *>(blk_dst[b]);
    const uint4 first = desc[static_cast<long long>(b) * P + p0];
    const uint4 last = desc[static_cast<long long>(b) * P + p1 - 1];
    const uint32_t r0 = first.w, r1 = last.w + last.x;         // the CTA's byte range in the block
    const bool staged = r1 - r0 <= static_cast<uint32_t>(kCompactBytes);
    const uint4 d = p < p1 ? desc[sid] : make_uint4(0u, 0u, 0u, 0u);
    const T *col = counts + static_cast<size_t>(b) * kScans * P + p;
    const uint32_t *sl = slots + static_cast<size_t>(sid) * kSlotWords;
    if (!staged) {
        if (d.x) {
            uint8_t *o = blk + d.w;
            uint32_t at, len;
            write_head<T>(o, col, P, d, at, len);
            const uint4 *s4 = reinterpret_cast<const uint4 *>(sl);
            for (uint32_t q = 0; q < len; q += 16) {
                const uint4 c = __ldcs(s4 + q / 16);
                const uint32_t wv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (q + i < len)
                        o[at + q + i] = static_cast<uint8_t>(wv[i >> 2] >> (8 * (i & 3)));
            }
        }
        return;
    }
    uint8_t *dst0 = blk + r0;
    const uint32_t mis = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(dst0) & 15u);
    const uint32_t span = mis + (r1 - r0);                      // staged bytes from the aligned start
    for (uint32_t c = threadIdx.x; c * 16 < span; c += kCompactThreads)
        reinterpret_cast<uint4 *>(s_buf)[c] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    uint32_t at = 0, len = 0;
    const uint32_t o = mis + (d.w - r0);
    if (d.x)
        write_head<T>(s_buf + o, col, P, d, at, len);
    uint32_t n_chunks;
    const uint32_t c0 = block_exclusive_scan((len + 15u) / 16u, s_warp, n_chunks);
    s_chunk0[threadIdx.x] = c0;
    s_at[threadIdx.x] = o + at;
    s_len[threadIdx.x] = len;
    __syncthreads();
    const uint4 *slot0 = reinterpret_cast<const uint4 *>(slots + static_cast<size_t>(static_cast<long long>(b) * P + p0) *
                                                                     kSlotWords);
    for (uint32_t cb = threadIdx.x; cb < n_chunks; cb += kCompactUnroll * kCompactThreads) {
        uint4 v[kCompactUnroll];
        int who[kCompactUnroll];
        uint32_t j[kCompactUnroll];
#pragma unroll
        for (int u = 0; u < kCompactUnroll; ++u) {
            const uint32_t c = cb + u * kCompactThreads;
            who[u] = -1;
            if (c < n_chunks) {
                // the stream whose chunks hold c: the last one starting at or before c
                int lo = 0, hi = kCompactThreads - 1;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (s_chunk0[mid] <= c)
                        lo = mid;
                    else
                        hi = mid - 1;
                }
                who[u] = lo;
                j[u] = c - s_chunk0[lo];
                v[u] = __ldcs(slot0 + static_cast<size_t>(lo) * (kSlotWords / 4) + j[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < kCompactUnroll; ++u) {
            if (who[u] < 0)
                continue;
            const uint32_t rem = s_len[who[u]] - 16u * j[u];   // >= 1
            uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            if (rem < 16u) {
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int keep = min(4, max(0, static_cast<int>(rem) - 4 * t));
                    w[t] = keep == 4 ? w[t] : (w[t] & ((1u << (8 * keep)) - 1u));
                }
            }
            const uint32_t a = s_at[who[u]] + 16u * j[u];
            const uint32_t m = (a & 3u) * 8u;
            uint32_t *wp = reinterpret_cast<uint32_t *>(s_buf + (a & ~3u));
#pragma unroll
            for (int t = 0; t < 5; ++t) {
                const uint32_t x = __funnelshift_l(t ? w[t - 1] : 0u, t < 4 ? w[t] : 0u, m);
                if (x)
                    atomicOr(wp + t, x);
            }
        }
    }
    __syncthreads();
    uint8_t *aligned = dst0 - mis;
    for (uint32_t c = threadIdx.x; c * 16 < span; c += kCompactThreads) {
        const uint32_t lo = c * 16, hi = lo + 16;
        if (lo >= mis && hi <= span) {
            *reinterpret_cast<uint4 *>(aligned + lo) = *reinterpret_cast<const uint4 *>(s_buf + lo);
        } else {
            for (uint32_t i = lo; i < hi && i < span; ++i)
                if (i >= mis)
                    aligned[i] = s_buf[i];
        }
    }
}

// ---------------------------------------------------------------------------
// a5: plan
// ---------------------------------------------------------------------------
constexpr int kPlanThreads = 256;

// Blocks [0, n_list_blocks) build the pixel list, one pixel per thread: each
// warp ballots its 32 pixels and the block reserves room for all its warps
// with one atomic per class.
// Pixels of the heavy class (decoded pair by pair) fill the list from the
// front (count[0]), light ones (empty, sparse, run-decoded) from the back
// (count[1], list[P-1], list[P-2], ...), so that warps meet one kind of work.
// Order inside a class does not matter to the sums (integer addition).
// Full query (mode 0): mask && valid; delta (1): pixels whose (mask && valid)
// changed against the stored baseline mask, leaving pixels flagged in bit 31;
// complement (2): the valid pixels outside the mask, all flagged.  Every
// thread then stores the new mask as the baseline.  Blocks past n_list_blocks initialise
// the rows: a full query zeroes the output and the kept image, a delta starts
// the output from the kept image, a complement query starts both from the
// cached full-detector image (the decode adds its terms to both).  The
// counter pair of the next query (count_next) is cleared here, so that no
// separate clear is needed between queries.
__global__ void __launch_bounds__(kPlanThreads) k_plan(const uint8_t *__restrict__ mask,
                                                      const uint8_t *__restrict__ valid,
                                                      const uint8_t *__restrict__ pclass,
                                                      uint8_t *__restrict__ base_mask, int P, int mode,
                                                      int n_list_blocks, uint32_t *__restrict__ list,
                                                      uint32_t *__restrict__ count,
                                                      uint32_t *__restrict__ count_next, uint4 *__restrict__ out,
                                                      uint4 *__restrict__ keep, long long n_vec,
                                                      const unsigned long long *__restrict__ total, int stride,
                                                      int out_bytes)
{
    // the decode that follows may start its prologue (table copy) now; it
    // waits for this grid's completion before it reads anything written here
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (blockIdx.x == 0 && threadIdx.x < 4)
        count_next[threadIdx.x] = 0u;
    if (static_cast<int>(blockIdx.x) < n_list_blocks) {
        constexpr int NW = kPlanThreads / 32;
        __shared__ uint32_t s_h[NW], s_l[NW], s_at[2];
        const int p = static_cast<int>(blockIdx.x) * kPlanThreads + static_cast<int>(threadIdx.x);
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        bool emit = false, light = false;
        uint32_t entry = 0;
        uint8_t mk = 0;
        if (p < P) {
            const bool ok = valid[p] != 0;
            mk = mask[p];
            const bool nw = ok && mk != 0;
            const bool od = ok && base_mask[p] != 0;
            if (mode == 0) {
                emit = nw;
                entry = static_cast<uint32_t>(p);
            } else if (mode == 1) {
                emit = nw != od;
                entry = static_cast<uint32_t>(p) | (od ? 0x80000000u : 0u);
            } else {
                // complement: the valid pixels outside the mask, subtracted
                emit = ok && mk == 0;
                entry = static_cast<uint32_t>(p) | 0x80000000u;
            }
            light = pclass[p] != 0;
            base_mask[p] = mk;
        }
        const unsigned bh = __ballot_sync(kFull, emit && !light);
        const unsigned bl = __ballot_sync(kFull, emit && light);
        if (lane == 0) {
            s_h[warp] = static_cast<uint32_t>(__popc(bh));
            s_l[warp] = static_cast<uint32_t>(__popc(bl));
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            // exclusive prefix over the warps, then one reservation per class
            uint32_t th = 0, tl = 0;
            for (int w = 0; w < NW; ++w) {
                const uint32_t a = s_h[w], c = s_l[w];
                s_h[w] = th;
                s_l[w] = tl;
                th += a;
                tl += c;
            }
            s_at[0] = th ? atomicAdd(count, th) : 0u;
            s_at[1] = tl ? atomicAdd(count + 1, tl) : 0u;
        }
        __syncthreads();
        const unsigned below = (1u << lane) - 1u;
        if (emit && !light)
            list[s_at[0] + s_h[warp] + __popc(bh & below)] = entry;
        if (emit && light)
            list[P - 1 - (s_at[1] + s_l[warp] + __popc(bl & below))] = entry;
        return;
    }
    const long long step = static_cast<long long>(gridDim.x - n_list_blocks) * blockDim.x;
    for (long long i = static_cast<long long>(blockIdx.x - n_list_blocks) * blockDim.x + threadIdx.x; i < n_vec;
         i += step) {
        if (mode == 0) {
            out[i] = make_uint4(0u, 0u, 0u, 0u);
            if (keep)
                keep[i] = make_uint4(0u, 0u, 0u, 0u);
        } else if (mode == 1) {
            out[i] = keep[i];
        } else {
            // complement: every row starts from the cached full-detector image of
            // its block (total is [B][512] uint64; row r holds block r * stride)
            const long long per = 16 / out_bytes;
            const long long e0 = i * per, row = e0 / kScans, col = e0 - row * kScans;
            const unsigned long long *t = total + (row * stride) * kScans + col;
            uint4 v;
            if (out_bytes == 4)
                v = make_uint4(static_cast<uint32_t>(t[0]), static_cast<uint32_t>(t[1]), static_cast<uint32_t>(t[2]),
                               static_cast<uint32_t>(t[3]));
            else
                v = make_uint4(static_cast<uint32_t>(t[0]), static_cast<uint32_t>(t[0] >> 32),
                               static_cast<uint32_t>(t[1]), static_cast<uint32_t>(t[1] >> 32));
            out[i] = v;
            keep[i] = v;
        }
    }
}

// ---------------------------------------------------------------------------
// a6: fused decode + masked reduce (the hot kernel)
// ---------------------------------------------------------------------------
// Persistent CTAs, one per SM; one 4 KB table per model (run-event tables of
// the low-dose models, decode tables of the others) lives in shared memory.
// Index items (whole pixel groups served from stored sums) go first.  Then the
// decode work, a 1-D list of warp tasks (touched block row, tile of 32 listed
// pixels), is cut into one contiguous share per CTA; its warps take tasks from
// a shared counter.  Each warp decodes its 32 streams (one per lane) 32 scans
// at a time and reduces them across the warp with redux.sync into the row's
// shared slot; the warp that finishes a row piece's last task adds the slot to
// the output with one global atomic per nonzero scan sum.
// Add v to a scan accumulator: an explicit shared-space reduction for the
// masked sum's accumulators (shared memory), a global atomic for the index
// build's.
template <bool SHARED>
__device__ __forceinline__ void acc_add(uint32_t *p, uint32_t v)
{
    if constexpr (SHARED)
        asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))), "r"(v)
                     : "memory");
    else
        atomicAdd(p, v);
}

// acc_add when `add` is nonzero, without a branch: a predicated reduction
// (the run-event loop's lanes add their rare nonzero counts at different
// events, so a branch per count diverges)
template <bool SHARED>
__device__ __forceinline__ void acc_add_if(uint32_t *p, uint32_t v, uint32_t add)
{
    if constexpr (SHARED)
        asm volatile("{\n\t"
                     ".reg .pred q;\n\t"
                     "setp.ne.u32 q, %2, 0;\n\t"
                     "@q red.shared.add.u32 [%0], %1;\n\t"
                     "}" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))),
                     "r"(v), "r"(add)
                     : "memory");
    else if (add)
        atomicAdd(p, v);
}

template <int W, bool DELTA, bool ROOMY = false, bool ACC_SHARED = false>
__device__ __forceinline__ void decode_task(const View &v, const uint32_t *s_dec, const uint32_t *dec_g,
                                            uint32_t skip_models, const uint32_t *list, uint32_t n,
                                            uint32_t n_l, int tile,
                                            long long b, uint32_t *acc, uint32_t *stage, uint32_t *cnt,
                                            uint64_t *bar, bool &ready, int lane, DevStatus *st)
{
    // tiles [0, tiles_h) cover the heavy entries list[0, n_h); the rest cover
    // the light entries list[P - n_l, P)
    const uint32_t n_h = n & 0xFFFFFFFFu;
    const uint32_t tiles_h = (n_h + 31u) >> 5;
    uint32_t idx;
    bool listed;
    if (static_cast<uint32_t>(tile) < tiles_h) {
        idx = static_cast<uint32_t>(tile) * 32u + static_cast<uint32_t>(lane);
        listed = idx < n_h;
    } else {
        idx = static_cast<uint32_t>(v.P) - n_l + (static_cast<uint32_t>(tile) - tiles_h) * 32u +
              static_cast<uint32_t>(lane);
        listed = idx < static_cast<uint32_t>(v.P);
    }
    const uint32_t e = listed ? __ldg(list + idx) : 0u;
    const int p = static_cast<int>(e & 0x7FFFFFFFu);
    listed = listed && p < v.P;     // the index build's lists hold padding slots (p >= P)
    const bool neg = DELTA && (e >> 31) != 0u;
    Stream S;
    S.form = kEmpty;
    S.model = 0;
    S.shift = 0;
    S.base = 0;
    S.c = 0;
    S.x = 0;
    S.x2 = 0;
    S.two = false;
    S.len = 0;
    bool ok = listed;
    if (ok)
        ok = locate(v, b, p, S.s, S.len, st);
    if (ok)
        ok = open_stream(S, W, st);
    if (!ok)
        S.form = kEmpty;
    if (!ready) {
        // first task of this thread: the tables must have landed (the stream
        // opens above overlapped their copy)
        if (!tables_wait(bar, st))
            S.form = kEmpty;
        ready = true;
    }

    const unsigned nact = __popc(__ballot_sync(kFull, listed));
    if (lane == 0) {
        if (tile == 0)
            atomicAdd(cnt, 1u);
        atomicAdd(cnt + 1, nact);
    }

    // low-dose paired streams (models dominated by the (0,0) symbol) are decoded
    // by runs after the per-scan loop instead of inside it.  Those models'
    // shared-memory slices hold their run tables; the rare stream of such a
    // model that also has a base or raw bits reads its decode table from
    // global memory (cached) instead.
    const bool run_model = (skip_models >> S.model) & 1u;
    const bool runs = S.form == kPaired && S.shift == 0 && S.base == 0u && run_model;
    const uint32_t *dec = (run_model ? dec_g : s_dec) + S.model * kStates;
    const bool dense_lane = (S.form == kPaired && !runs) || S.form == kLiteral || S.form == kConstant;
    // A warp with a paired lane that needs the general step (a base or raw
    // low bits: one count of 16 or more in a low-count stream is enough) runs
    // the general step on all its paired lanes: with both kinds in one warp
    // the fast loop and the general loop would run one after the other.
    const bool plain_warp = __all_sync(kFull, !(S.form == kPaired && !runs) || (S.shift == 0 && S.base == 0u));
    // In the kernels launched with room for more registers per thread (uint8
    // deltas, every uint16 query), a warp whose pair-by-pair lanes all use
    // two-state models takes the two-state loop even when some lanes carry a
    // base or raw low bits (one count of 16 or more in a low-count stream is
    // enough; every high-dose uint16 pixel): those are added per pair after the
    // table steps, each half on its own for uint16 (a value is at most 65535).
    const bool two_lane = S.form == kPaired && !runs && S.two;
    bool fast = plain_warp && two_lane && S.shift == 0 && S.base == 0u;
    bool raw_warp = false;
    // uint8: when exactly one lane of such a warp carries raw low bits, the whole warp
    // reads them: lane l holds words l, l + 32 and l + 64 of that lane's raw
    // section (at most 4 bits x 512 scans + the lead), and per 32-scan segment
    // each lane extracts the low bits of its own scan.  The raw lane's table
    // steps are shifted like every other lane's; its low bits join the scan
    // sums after the warp reduction.  (The raw lane alone would spend ~16
    // instructions per pair on them, the whole warp waiting.)
    int coop_r = -1;
    uint32_t rw0 = 0u, rw1 = 0u, rw2 = 0u, r_lead = 0u, r_shift = 0u;
    bool r_neg = false;
    if constexpr (ROOMY) {
        const bool all_two = __all_sync(kFull, !(S.form == kPaired && !runs) || S.two);
        raw_warp = __any_sync(kFull, two_lane && (S.shift != 0 || S.base != 0u));
        fast = all_two && two_lane;
        const unsigned rm = __ballot_sync(kFull, all_two && two_lane && S.shift != 0);
        if (W == 1 && __popc(rm) == 1) {
            coop_r = __ffs(rm) - 1;
            const unsigned long long f =
                __shfl_sync(kFull, reinterpret_cast<unsigned long long>(S.br.first), coop_r);
            const uint32_t li = __shfl_sync(kFull, S.br.li, coop_r);
            r_lead = __shfl_sync(kFull, static_cast<uint32_t>(S.br.lead), coop_r);
            r_shift = __shfl_sync(kFull, static_cast<uint32_t>(S.shift), coop_r);
            r_neg = __shfl_sync(kFull, neg ? 1u : 0u, coop_r) != 0u;
            const uint32_t *fw = reinterpret_cast<const uint32_t *>(f);
            rw0 = __ldg(fw + min(static_cast<uint32_t>(lane), li));
            rw1 = __ldg(fw + min(static_cast<uint32_t>(lane) + 32u, li));
            rw2 = __ldg(fw + min(static_cast<uint32_t>(lane) + 64u, li));
        }
    }
    uint32_t over = 0;
    // warps whose lanes hold only empty, sparse or run-decoded streams skip the per-scan loop
    const bool dense = __any_sync(kFull, dense_lane);

    // A uint16 warp whose dense lanes are all two-state paired streams (with or,
    // in the kernels with room for it, without a base and raw low bits) or small
    // constants takes the packed path as well: a segment whose values all stay
    // below kPackMax + 1 is reduced in packed halves, any other segment scan by
    // scan (32 lanes x kPackMax must fit a 16-bit half).
    constexpr uint32_t kPackMax = W == 1 ? 255u : 2047u;
    const bool packed = W == 1 || __all_sync(kFull, !dense_lane || fast || (S.form == kConstant && S.c <= 255u));
    if (packed) {
        // counts fit 16-bit halves: pack scans (2j, 2j+1) into one word; a
        // leaving pixel contributes kPackMax - v per half and the warp subtracts
        // kPackMax x (number of such lanes) afterwards.
        const bool packed_src = dense_lane;
        const uint32_t flip = (neg && packed_src) ? (kPackMax | (kPackMax << 16)) : 0u;
        const uint32_t corr = kPackMax * static_cast<uint32_t>(__popc(__ballot_sync(kFull, neg && packed_src)));
        const uint32_t cpk = S.form == kConstant ? (S.c | (S.c << 16)) : 0u;
        const uint32_t dec_sa = static_cast<uint32_t>(__cvta_generic_to_shared(dec));
        for (int seg = 0; seg < (dense ? 16 : 0); ++seg) {
            uint32_t pk[16];
            if (fast) {
                // two interleaved states (fast streams use models 8-31, spec S3):
                // both table loads first, then the bits of pair A, then pair B
#pragma unroll
                for (int jj = 0; jj < 16; jj += 2) {
                    const uint32_t ea = tab_load(S.x, dec_sa);
                    const uint32_t eb = tab_load(S.x2, dec_sa);
                    // top-ups before pairs 0, 3, 6, 9, 12, 15: <= 30 bits per 3 pairs
                    if (jj % 3 == 0 && S.bt.n < 30)
                        S.bt.refill();
                    pk[jj] = consume(ea, S.x, S.bt.lo, S.bt.hi, S.bt.n);
                    if ((jj + 1) % 3 == 0 && S.bt.n < 30)
                        S.bt.refill();
                    pk[jj + 1] = consume(eb, S.x2, S.bt.lo, S.bt.hi, S.bt.n);
                }
                if constexpr (ROOMY) {
                  if (W == 1 && raw_warp && coop_r >= 0) {
                    // v = base + (hi << shift), both halves at once; the raw lane's
                    // low bits are added after the reduction (below)
                    const uint32_t bpk = S.base | (S.base << 16);
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        const uint32_t v = (pk[jj] << S.shift) + bpk;
                        over |= (v & 0xFFFFu) | (v >> 16);
                        pk[jj] = v;
                    }
                  } else if (raw_warp && W == 1) {
                    // v = base + (hi << shift | lo), both halves at once
                    const uint32_t m = (1u << S.shift) - 1u;
                    const uint32_t bpk = S.base | (S.base << 16);
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        if (S.br.n < 2 * S.shift)
                            S.br.refill();
                        const uint32_t lo = S.br.get(2 * S.shift);
                        const uint32_t v = ((pk[jj] << S.shift) | (lo & m) | (((lo >> S.shift) & m) << 16)) + bpk;
                        over |= (v & 0xFFFFu) | (v >> 16);
                        pk[jj] = v;
                    }
                  } else if (raw_warp) {
                    // uint16: each half on its own (a malformed stream's value
                    // past 65535 must not carry into the other half unseen)
                    const uint32_t m = (1u << S.shift) - 1u;
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        if (S.br.n < 2 * S.shift)
                            S.br.refill();
                        const uint32_t lo = S.br.get(2 * S.shift);
                        const uint32_t va = (((pk[jj] & 0xFFFFu) << S.shift) | (lo & m)) + S.base;
                        const uint32_t vb = (((pk[jj] >> 16) << S.shift) | ((lo >> S.shift) & m)) + S.base;
                        over |= va | vb;
                        pk[jj] = va | (vb << 16);
                    }
                  }
                }
            } else if (S.form == kPaired && !runs) {
                uint32_t vv[32];
                paired_segment(S, dec, vv, over);
#pragma unroll
                for (int jj = 0; jj < 16; ++jj)
                    pk[jj] = vv[2 * jj] | (vv[2 * jj + 1] << 16);
            } else if (W == 1 && S.form == kLiteral) {
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    if (S.bt.n < 16)
                        S.bt.refill();
                    const uint32_t a = S.bt.get(8);
                    const uint32_t c = S.bt.get(8);
                    pk[jj] = a | (c << 16);
                }
            } else {
#pragma unroll
                for (int jj = 0; jj < 16; ++jj)
                    pk[jj] = cpk;
            }
            uint32_t lo_add = 0u;
            if constexpr (W == 1 && ROOMY) {
                if (coop_r >= 0) {
                    // (warp-uniform: every lane takes part, whatever its own stream)
                    // the raw lane's value of scan seg * 32 + lane without its low
                    // bits, through shared memory; then the low bits of that scan
                    // from the words the lanes hold, and the full value's range check
                    if (lane == coop_r) {
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj)
                            stage[jj] = pk[jj];
                    }
                    __syncwarp();
                    const uint32_t vw = stage[lane >> 1];
                    __syncwarp();
                    const uint32_t vp = (lane & 1) ? (vw >> 16) : (vw & 0xFFFFu);
                    const uint32_t bit = r_lead + static_cast<uint32_t>(seg * 32 + lane) * r_shift;
                    const uint32_t k0 = bit >> 5, k1 = k0 + 1u;
                    const uint32_t a0 = __shfl_sync(kFull, rw0, static_cast<int>(k0 & 31u));
                    const uint32_t a1 = __shfl_sync(kFull, rw1, static_cast<int>(k0 & 31u));
                    const uint32_t a2 = __shfl_sync(kFull, rw2, static_cast<int>(k0 & 31u));
                    const uint32_t b0 = __shfl_sync(kFull, rw0, static_cast<int>(k1 & 31u));
                    const uint32_t b1 = __shfl_sync(kFull, rw1, static_cast<int>(k1 & 31u));
                    const uint32_t b2 = __shfl_sync(kFull, rw2, static_cast<int>(k1 & 31u));
                    const uint32_t w0 = k0 < 32u ? a0 : (k0 < 64u ? a1 : a2);
                    const uint32_t w1 = k1 < 32u ? b0 : (k1 < 64u ? b1 : b2);
                    const uint32_t lo = __funnelshift_r(w0, w1, bit & 31u) & ((1u << r_shift) - 1u);
                    if (vp + lo > 0xFFu)
                        report(st, kErrValue);
                    lo_add = r_neg ? 0u - lo : lo;
                }
            }
            if constexpr (W == 2 && ROOMY) {
                // a segment with a value above kPackMax is reduced scan by scan
                uint32_t so = 0u;
#pragma unroll
                for (int jj = 0; jj < 16; ++jj)
                    so |= pk[jj];
                if (__any_sync(kFull, ((so | (so >> 16)) & 0xFFFFu) > kPackMax)) {
                    uint32_t mine = 0u;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const uint32_t v = (i & 1) ? (pk[i >> 1] >> 16) : (pk[i >> 1] & 0xFFFFu);
                        const uint32_t r = __reduce_add_sync(kFull, neg ? 0u - v : v);
                        if (lane == i)
                            mine = r;
                    }
                    if (mine)
                        acc_add<ACC_SHARED>(acc + seg * 32 + lane, mine);
                    continue;
                }
            }
            // warp sums of the 16 packed pairs are warp-uniform: one lane
            // parks them in shared memory, every lane then takes its scan
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const uint32_t r = __reduce_add_sync(kFull, DELTA ? (pk[jj] ^ flip) : pk[jj]);
                if (lane == 0)
                    stage[jj] = r;
            }
            __syncwarp();
            uint32_t mine = stage[lane >> 1];
            __syncwarp();
            mine = ((lane & 1) ? (mine >> 16) : (mine & 0xFFFFu)) - (DELTA ? corr : 0u) + lo_add;
            if (mine)
                acc_add<ACC_SHARED>(acc + seg * 32 + lane, mine);
        }
    } else {
        const uint32_t sgn = neg ? 0xFFFFFFFFu : 0u;       // v -> (v ^ sgn) - sgn negates
        for (int seg = 0; seg < (dense ? 16 : 0); ++seg) {
            uint32_t vv[32];
            if (S.form == kPaired && !runs) {
                paired_segment(S, dec, vv, over);
            } else if (S.form == kLiteral) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if (S.bt.n < 16)
                        S.bt.refill();
                    vv[i] = S.bt.get(16);
                }
            } else {
                const uint32_t c = S.form == kConstant ? S.c : 0u;
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    vv[i] = c;
            }
            uint32_t mine = 0;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const uint32_t r = __reduce_add_sync(kFull, DELTA ? (vv[i] ^ sgn) - sgn : vv[i]);
                if (lane == i)
                    mine = r;
            }
            if (mine)
                acc_add<ACC_SHARED>(acc + seg * 32 + lane, mine);
        }
    }

    if (runs) {
        // One event per iteration, one shared-memory read: jump the run of
        // zero-bit (0,0) steps from the current state (possibly empty), then
        // take the ordinary step at the slot reached, adding its nonzero
        // counts to their scans.  A run that passes pair 255 cannot end in the
        // final state 1024 (that state reads bits), so it marks the stream
        // malformed; a run that ends exactly at pair 256 leaves the stream in
        // the slot it reached, which the end check then requires to be 0.
        // Each iteration advances j, so the loop ends.
        // The entry of the next event is read before this event's counts are
        // added (predicated, no branch): with both, the loop takes ~10 % less
        // time on low-dose streams than reading it after divergent adds.
        const uint32_t rt_sa = static_cast<uint32_t>(__cvta_generic_to_shared(s_dec + S.model * kStates));
        int j = 0;
        bool bad = false;
        uint32_t t = tab_load_ordered(S.x, rt_sa);
        while (j < kPairs) {
            j += static_cast<int>((t >> 14) & 63u);
            if (j >= kPairs) {
                bad = j > kPairs;
                S.x = (t >> 28) & 1u;
                break;
            }
            if (S.bt.n < 10)
                S.bt.refill();
            S.x = (t & 1023u) | S.bt.get(static_cast<int>((t >> 10) & 15u));
            const uint32_t tn = tab_load_ordered(S.x, rt_sa);
            const uint32_t a = (t >> 20) & 15u, c = (t >> 24) & 15u;
            acc_add_if<ACC_SHARED>(acc + 2 * j, neg ? 0u - a : a, a);
            acc_add_if<ACC_SHARED>(acc + 2 * j + 1, neg ? 0u - c : c, c);
            ++j;
            t = tn;
        }
        if (bad)
            report(st, kErrState);
        else
            close_paired(S, st);
    } else if (S.form == kPaired) {
        if (over > (W == 1 ? 0xFFu : 0xFFFFu)) {
            report(st, kErrValue);
        }
        close_paired(S, st);
    } else if (S.form == kSparse) {
        // sparse: scatter the nonzeros (positions strictly ascending, values nonzero)
        int prev = -1;
        bool bad = false;
        for (uint32_t k = 0; k < S.c; ++k) {
            if (S.bt.n < 9)
                S.bt.refill();
            const int pos = static_cast<int>(S.bt.get(9));
            if (S.br.n < 16)
                S.br.refill();
            const uint32_t val = S.br.get(8 * W);
            if (pos <= prev || val == 0u) {
                bad = true;
                break;
            }
            prev = pos;
            acc_add<ACC_SHARED>(acc + pos, neg ? 0u - val : val);
        }
        if (bad) {
            report(st, kErrSparse);
        } else {
            const int pad = static_cast<int>(((9u * S.c + 7u) / 8u) * 8u - 9u * S.c);
            if (pad) {
                if (S.bt.n < pad)
                    S.bt.refill();
                if (S.bt.get(pad) != 0u)
                    report(st, kErrPad);
            }
        }
    }
}

// One index task: items [c * K, ...) of the item list, for block
// b (output row `row`).  Item: bit 31 = subtract, bit 30 = root level, bits
// 0-29 = group number within its level.  A group's 512 sums are stored with
// one width per (block, group) (desc bits 30-31: 0 = all zero, 1/2/3 = 1, 2
// or 4 bytes per sum; bits 0-29 = byte offset in the block's index bytes).
// Lane l adds the sums of scans l, l + 32, ..., l + 480 (coalesced reads).
// A task's partial sums stay below 2^31 in magnitude (K = 32 groups of at
// most 1024 8-bit counts, or 16 groups of 16-bit counts), so a 64-bit output
// takes them sign-extended.
template <int W>
__device__ __forceinline__ void index_task(const IndexView &ix, long long b, uint32_t i0, uint32_t cnt, long long row,
                                           void *out, void *keep, int out_bytes, int lane)
{
    uint32_t acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
        acc[j] = 0u;
    // lane i fetches item i of the task and its descriptor: one round trip
    // for all of them (cnt <= 32)
    uint32_t my_it = 0u, my_d = 0u;
    if (static_cast<uint32_t>(lane) < cnt) {
        my_it = __ldg(ix.items + i0 + lane);
        const int g = static_cast<int>(my_it & 0x3FFFFFFFu) + (((my_it >> 30) & 1u) ? ix.L : 0);
        my_d = __ldg(ix.desc + static_cast<long long>(b) * ix.G + g);
    }
    const unsigned long long base = __ldg(ix.base + b);
    // scans lane, lane + 32, ... of item i (zeros for an all-zero group); the
    // returned mask negates a subtracted item's sums
    auto fetch = [&](uint32_t i, uint32_t (&v)[16]) {
        const uint32_t d = __shfl_sync(kFull, my_d, static_cast<int>(i));
        const uint32_t it = __shfl_sync(kFull, my_it, static_cast<int>(i));
        const uint32_t code = d >> 30;
        const unsigned long long a = base + (d & 0x3FFFFFFFu);
        if (code == 1u) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
                v[j] = __ldg(reinterpret_cast<const uint8_t *>(a) + lane + 32 * j);
        } else if (code == 2u) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
                v[j] = __ldg(reinterpret_cast<const uint16_t *>(a) + lane + 32 * j);
        } else if (code == 3u) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
                v[j] = __ldg(reinterpret_cast<const uint32_t *>(a) + lane + 32 * j);
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
                v[j] = 0u;
        }
        return (it >> 31) ? 0xFFFFFFFFu : 0u;     // v -> (v ^ sgn) - sgn negates
    };
    // two items at a time: the loads of both are in flight before either is added
    for (uint32_t i = 0; i < cnt; i += 2) {
        uint32_t va[16], vb[16];
        const uint32_t sa = fetch(i, va);
        uint32_t sb = 0u;
        if (i + 1 < cnt) {
            sb = fetch(i + 1, vb);
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
                vb[j] = 0u;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j)
            acc[j] += ((va[j] ^ sa) - sa) + ((vb[j] ^ sb) - sb);
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        if (acc[j] == 0u)
            continue;
        const long long o = row * kScans + lane + 32 * j;
        if (out_bytes == 4) {
            atomicAdd(reinterpret_cast<unsigned int *>(out) + o, acc[j]);
            if (keep)
                atomicAdd(reinterpret_cast<unsigned int *>(keep) + o, acc[j]);
        } else {
            const unsigned long long wide = static_cast<unsigned long long>(static_cast<long long>(static_cast<int>(acc[j])));
            atomicAdd(reinterpret_cast<unsigned long long *>(out) + o, wide);
            if (keep)
                atomicAdd(reinterpret_cast<unsigned long long *>(keep) + o, wide);
        }
    }
}

constexpr int kMaxSlots = 8;    // block rows one CTA range may touch (shared accumulators)

// a / b for 0 <= a, 0 < b < 2^32: a 32-bit division when a fits in 32 bits
// (task numbers of every realistic query), the 64-bit one otherwise
__device__ __forceinline__ long long qdiv(long long a, long long b)
{
    if ((static_cast<unsigned long long>(a) >> 32) == 0ull)
        return static_cast<long long>(static_cast<uint32_t>(a) / static_cast<uint32_t>(b));
    return a / b;
}

template <int W, int THREADS, bool DELTA>
__global__ void __launch_bounds__(THREADS, 1) k_decode_reduce(View v, const uint32_t *__restrict__ dec_g,
                                                             const uint32_t *__restrict__ runs_g,
                                                             uint32_t skip_models, int skip_count,
                                                             const uint32_t *__restrict__ list,
                                                             const uint32_t *__restrict__ count, int stride,
                                                             long long rows, void *__restrict__ out,
                                                             void *__restrict__ keep, int out_bytes,
                                                             IndexView ix, DevStatus *__restrict__ st)
{
    constexpr int MAXW = THREADS / 32;
    // shared memory: one 4 KB table per model (the run tables of the first
    // skip_count models, the decode tables of the others) | per-warp staging |
    // kMaxSlots per-row scan accumulators
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t *s_dec = smem;
    uint32_t *s_stage = smem + kModels * kStates;   // 16 words per warp
    uint32_t *s_acc = s_stage + MAXW * 16;
    __shared__ __align__(8) uint64_t s_bar;
    if (threadIdx.x == 0)
        tables_start(&s_bar, s_dec, dec_g, runs_g, skip_count);
    bool ready = false;
    // per-CTA counters (rows, streams), added to the status once at the end
    __shared__ uint32_t s_cnt[2];
    if (threadIdx.x < 2)
        s_cnt[threadIdx.x] = 0u;

    // launched as a programmatic dependent of the plan: everything above only
    // touched shared memory and the constant tables; wait here until the plan
    // grid has finished and its list, counts and rows are visible
    for (int i = threadIdx.x; i < kMaxSlots * kScans; i += THREADS)
        s_acc[i] = 0u;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const uint32_t n = __ldg(count);          // heavy entries, list[0, n)
    const uint32_t n_l = __ldg(count + 1);    // light entries, list[P - n_l, P)
    const long long tiles = ((n + 31u) >> 5) + ((n_l + 31u) >> 5);
    const long long total = rows * tiles;
    const int warp0 = threadIdx.x >> 5, lane0 = threadIdx.x & 31;
    // Each CTA owns one contiguous share [T0, T1) of the tasks (row-major:
    // row, then tile); its warps take the next task from a shared counter as
    // they finish, with no barrier between tasks.  Scan sums of a row gather
    // in one of kMaxSlots shared slots; the warp that completes a row's last
    // task in this share adds the slot to the output and frees it for the
    // row kMaxSlots later.  Slots are 32-bit, so a row is cut into pieces of
    // at most F tasks (F * 32 pixels of full-scale counts stay below 2^31 in
    // magnitude); a piece ("vrow") is the unit that owns a slot.
    constexpr long long kMaxCount = W == 1 ? 255 : 65535;
    constexpr long long F = 0x7FFFFFFFll / (32 * kMaxCount);
    const long long nch = (tiles + F - 1) / F;              // pieces per row
    const long long T0 = qdiv(total * blockIdx.x, gridDim.x), T1 = qdiv(total * (blockIdx.x + 1), gridDim.x);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto vrow_of = [&](long long t) {
        const long long row = qdiv(t, tiles);
        return row * nch + (t - row * tiles) / F;
    };
    // tasks of piece vr inside [T0, T1)
    auto piece_tasks = [&](long long vr) {
        const long long row = qdiv(vr, nch), c = vr - row * nch;
        const long long a = row * tiles + c * F, b = row * tiles + min((c + 1) * F, tiles);
        return max(0ll, min(b, T1) - max(a, T0));
    };
    // A share whose pieces all hold a slot from the start may take its tasks
    // in any order.  It takes the heavy tiles of all its rows first, then the
    // light ones: a warp that finishes early and takes a second task then
    // takes a short one, instead of starting a heavy tile late.
    const long long th = static_cast<long long>((n + 31u) >> 5);
    const bool heavy_first = T1 > T0 && th > 0 && th < tiles && vrow_of(T1 - 1) - vrow_of(T0) < kMaxSlots;
    auto task_at = [&](long long k) {       // the k-th task of the share in that order
        const long long r0 = qdiv(T0, tiles), r1 = qdiv(T1 - 1, tiles);
        for (int pass = 0; pass < 2; ++pass)
            for (long long r = r0; r <= r1; ++r) {
                const long long lo = r == r0 ? T0 - r * tiles : 0, hi = r == r1 ? T1 - r * tiles : tiles;
                const long long a = pass ? max(lo, th) : lo, b = pass ? hi : min(hi, th);
                if (k < b - a)
                    return r * tiles + a + k;
                k -= max(0ll, b - a);
            }
        return T1;
    };
    __shared__ unsigned long long s_next;
    __shared__ long long s_owner[kMaxSlots];
    __shared__ uint32_t s_left[kMaxSlots];
    __shared__ int s_abort;                   // set once a wait ran out: the CTA stops taking tasks
    if (threadIdx.x == 0) {
        s_next = static_cast<unsigned long long>(T0 + MAXW);
        s_abort = 0;
    }
    if (threadIdx.x < kMaxSlots && T1 > T0) {
        const long long v0 = vrow_of(T0);
        const long long vr = v0 + ((threadIdx.x - v0) & (kMaxSlots - 1));
        s_owner[threadIdx.x] = vr;
        s_left[threadIdx.x] = static_cast<uint32_t>(vr <= vrow_of(T1 - 1) ? piece_tasks(vr) : 0);
    }
    __syncthreads();
    if (ix.desc != nullptr) {
        // index items (whole groups inside the mask, or inside its change),
        // before the warp's decode tasks and with no barrier between the two:
        // K per task, each lane adding the groups' stored sums of scans lane,
        // lane + 32, ...; the sums go straight to the output.  K is at most 32
        // (16 for 16-bit counts, so that K root sums stay below 2^31) and is
        // lowered, down to 4, until the tasks fill the grid's warps: a task's
        // items are read two at a time, so its time grows with K
        const uint32_t n_it = __ldg(count + 2);
        constexpr uint32_t kKMax = W == 1 ? 32u : 16u;
        const long long want = (static_cast<long long>(n_it) * rows + gridDim.x * MAXW - 1) / (gridDim.x * MAXW);
        const uint32_t K = static_cast<uint32_t>(max(4ll, min(static_cast<long long>(kKMax), want)));
        const long long chunks = (n_it + K - 1) / K;
        const long long itotal = rows * chunks;
        const long long I0 = qdiv(itotal * blockIdx.x, gridDim.x), I1 = qdiv(itotal * (blockIdx.x + 1), gridDim.x);
        for (long long t = I0 + warp0; t < I1; t += MAXW) {
            const long long row = qdiv(t, chunks);
            const uint32_t i0 = static_cast<uint32_t>(t - row * chunks) * K;
            index_task<W>(ix, row * stride, i0, min(K, n_it - i0), row, out, keep, out_bytes, lane0);
        }
    }
    // warp w takes task w of the share first (in heavy-first order the heavy
    // tiles go to warps 0, 1, 2, ..., spread evenly over the SM's four
    // schedulers), then the next from the counter
    bool first_task = true;
    while (true) {
        long long t = 0;
        if (lane == 0) {
            t = *reinterpret_cast<volatile int *>(&s_abort)
                    ? T1
                    : (first_task ? T0 + warp : static_cast<long long>(atomicAdd(&s_next, 1ull)));
            if (heavy_first && t < T1)
                t = task_at(t - T0);
        }
        first_task = false;
        t = __shfl_sync(kFull, t, 0);
        if (t >= T1)
            break;
        const long long row = qdiv(t, tiles);
        const int tile = static_cast<int>(t - row * tiles);
        const long long vr = row * nch + tile / F;
        const int slot = static_cast<int>(vr & (kMaxSlots - 1));
        // the slot may still hold the piece kMaxSlots earlier: wait (bounded)
        // until its last warp has emptied it.  That piece's tasks were all
        // taken before this one, so the wait ends.
        bool ok = true;
        if (lane == 0) {
            uint32_t it = 0;
            while (*reinterpret_cast<volatile long long *>(&s_owner[slot]) != vr) {
                if (++it > kWaitLimit) {
                    atomicOr(&st->flags, kErrWait);
                    *reinterpret_cast<volatile int *>(&s_abort) = 1;
                    ok = false;
                    break;
                }
                __nanosleep(32);
            }
        }
        ok = __shfl_sync(kFull, ok, 0);
        // a wait that ran out leaves the slot to its owner: this warp neither
        // decodes nor counts the task (the query reports QEM_ERR_TIMEOUT), so
        // no other piece's sums are flushed into this row
        if (!ok)
            continue;
        decode_task<W, DELTA, (THREADS <= 512 && (DELTA || W == 2)), true>(v, s_dec, dec_g, skip_models, list, n, n_l, tile,
                                                               row * stride, s_acc + slot * kScans, s_stage + warp * 16,
                                                               s_cnt, &s_bar, ready, lane, st);
        // this warp's slot additions happen before its count
        __threadfence_block();
        __syncwarp();
        uint32_t left = 0;
        if (lane == 0)
            left = atomicSub(&s_left[slot], 1u);
        left = __shfl_sync(kFull, left, 0);
        if (left == 1u) {
            __threadfence_block();
            uint32_t *acc = s_acc + slot * kScans;
            for (int i = lane; i < kScans; i += 32) {
                const uint32_t val = acc[i];
                if (val) {
                    acc[i] = 0u;
                    const long long o = row * kScans + i;
                    if (out_bytes == 4) {
                        atomicAdd(reinterpret_cast<unsigned int *>(out) + o, val);
                        if (keep)
                            atomicAdd(reinterpret_cast<unsigned int *>(keep) + o, val);
                    } else {
                        const unsigned long long wide =
                            static_cast<unsigned long long>(static_cast<long long>(static_cast<int>(val)));
                        atomicAdd(reinterpret_cast<unsigned long long *>(out) + o, wide);
                        if (keep)
                            atomicAdd(reinterpret_cast<unsigned long long *>(keep) + o, wide);
                    }
                }
            }
            __threadfence_block();
            __syncwarp();
            if (lane == 0) {
                const long long nv = vr + kMaxSlots;
                s_left[slot] = static_cast<uint32_t>(nv <= vrow_of(T1 - 1) ? piece_tasks(nv) : 0);
                __threadfence_block();
                *reinterpret_cast<volatile long long *>(&s_owner[slot]) = nv;
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // a CTA leaves only after its table copy has landed (CTAs without
        // tasks never waited on it)
        if (!ready)
            tables_wait(&s_bar, st);
        if (s_cnt[0] | s_cnt[1]) {
            atomicAdd(&st->rows, static_cast<unsigned long long>(s_cnt[0]));
            atomicAdd(&st->streams, static_cast<unsigned long long>(s_cnt[1]));
        }
    }
}

// ---------------------------------------------------------------------------
// masked moments (fused CoM / DPC numerators and denominator)
// ---------------------------------------------------------------------------
// For every touched block row and scan: sum of x * wr[p], of x * wc[p] and of
// x over the listed pixels (the plan's list of mask && valid pixels), exact in
// int64.  One CTA owns a row at a time (its warps take the row's tiles from a
// shared counter), so the row is written with plain stores.  Dense forms go
// through warp reductions of 32-bit partial sums (for 16-bit counts the value
// is split in bytes, so every partial sum stays below 2^31 for |w| < 2^18);
// sparse streams scatter their nonzeros into the row with shared atomics.
// Low-dose paired streams are decoded by run events (the run tables of those
// models in shared memory, as in the masked sum) and scatter their nonzero
// counts; other paired streams use the general decode.
template <int W>
__global__ void __launch_bounds__(512, 1) k_moments(View v, const uint32_t *__restrict__ dec_g,
                                                   const uint32_t *__restrict__ runs_g, uint32_t skip_models,
                                                   int skip_count, const uint32_t *__restrict__ list,
                                                   const uint32_t *__restrict__ count,
                                                   const int32_t *__restrict__ weights, int stride, long long rows,
                                                   long long *__restrict__ out, DevStatus *__restrict__ st)
{
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t *s_dec = smem;
    unsigned long long *s_acc = reinterpret_cast<unsigned long long *>(smem + kModels * kStates);  // [3][512]
    __shared__ unsigned s_next;
    // the run-event tables of the low-dose models, then the other decode tables
    for (int i = threadIdx.x; i < kModels * kStates / 4; i += blockDim.x)
        reinterpret_cast<uint4 *>(s_dec)[i] = i < skip_count * kStates / 4
                                                  ? __ldg(reinterpret_cast<const uint4 *>(runs_g) + i)
                                                  : __ldg(reinterpret_cast<const uint4 *>(dec_g) + i);
    for (int i = threadIdx.x; i < 3 * kScans; i += blockDim.x)
        s_acc[i] = 0ull;
    const uint32_t n = __ldg(count), n_l = __ldg(count + 1);
    const uint32_t tiles_h = (n + 31u) >> 5;
    const uint32_t tiles = tiles_h + ((n_l + 31u) >> 5);
    const int lane = threadIdx.x & 31;
    const long long P = v.P;
    for (long long row = blockIdx.x; row < rows; row += gridDim.x) {
        if (threadIdx.x == 0)
            s_next = 0u;
        __syncthreads();
        const long long b = row * stride;
        while (true) {
            unsigned tile = 0;
            if (lane == 0)
                tile = atomicAdd(&s_next, 1u);
            tile = __shfl_sync(kFull, tile, 0);
            if (tile >= tiles)
                break;
            uint32_t idx;
            bool listed;
            if (tile < tiles_h) {
                idx = tile * 32u + static_cast<uint32_t>(lane);
                listed = idx < n;
            } else {
                idx = static_cast<uint32_t>(P) - n_l + (tile - tiles_h) * 32u + static_cast<uint32_t>(lane);
                listed = idx < static_cast<uint32_t>(P);
            }
            const int p = listed ? static_cast<int>(__ldg(list + idx) & 0x7FFFFFFFu) : 0;
            const long long wr = listed ? __ldg(weights + p) : 0, wc = listed ? __ldg(weights + P + p) : 0;
            Stream S;
            S.form = kEmpty;
            S.model = 0;
            S.shift = 0;
            S.base = 0;
            S.c = 0;
            S.x = 0;
            S.x2 = 0;
            S.two = false;
            S.len = 0;
            bool ok = listed;
            if (ok)
                ok = locate(v, b, p, S.s, S.len, st);
            if (ok)
                ok = open_stream(S, W, st);
            if (!ok)
                S.form = kEmpty;
            // low-dose paired streams: run events scattered after the dense loop
            const bool run_model = (skip_models >> S.model) & 1u;
            const bool runs = S.form == kPaired && S.shift == 0 && S.base == 0u && run_model;
            const bool dense_lane = (S.form == kPaired && !runs) || S.form == kLiteral || S.form == kConstant;
            const bool dense = __any_sync(kFull, dense_lane);
            const uint32_t *dec = (run_model ? dec_g : s_dec) + S.model * kStates;
            // a warp whose pair-by-pair lanes are all two-state streams without
            // base or raw bits runs their interleaved table steps (models 8-31,
            // tables in shared memory) instead of the general step
            const bool two_plain = S.form == kPaired && !runs && S.two && S.shift == 0 && S.base == 0u;
            const bool fast_warp = __all_sync(kFull, !(S.form == kPaired && !runs) || two_plain);
            const uint32_t dec_sa = static_cast<uint32_t>(__cvta_generic_to_shared(s_dec + S.model * kStates));
            uint32_t over = 0;
            for (int seg = 0; seg < (dense ? 16 : 0); ++seg) {
                uint32_t vv[32];
                if (fast_warp && two_plain) {
#pragma unroll
                    for (int jj = 0; jj < 16; jj += 2) {
                        const uint32_t ea = tab_load(S.x, dec_sa);
                        const uint32_t eb = tab_load(S.x2, dec_sa);
                        if (jj % 3 == 0 && S.bt.n < 30)
                            S.bt.refill();
                        const uint32_t pa = consume(ea, S.x, S.bt.lo, S.bt.hi, S.bt.n);
                        if ((jj + 1) % 3 == 0 && S.bt.n < 30)
                            S.bt.refill();
                        const uint32_t pb = consume(eb, S.x2, S.bt.lo, S.bt.hi, S.bt.n);
                        vv[2 * jj] = pa & 0xFFFFu;
                        vv[2 * jj + 1] = pa >> 16;
                        vv[2 * jj + 2] = pb & 0xFFFFu;
                        vv[2 * jj + 3] = pb >> 16;
                    }
                } else if (S.form == kPaired && !runs) {
                    paired_segment(S, dec, vv, over);
                } else if (S.form == kLiteral) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        if (S.bt.n < 16)
                            S.bt.refill();
                        vv[i] = S.bt.get(8 * W);
                    }
                } else {
                    const uint32_t c = S.form == kConstant ? S.c : 0u;
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        vv[i] = c;
                }
                long long m0 = 0, m1 = 0, m2 = 0;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int x0 = static_cast<int>(vv[i]);
                    int a0 = __reduce_add_sync(kFull, x0);
                    long long a1, a2;
                    if (W == 1) {
                        a1 = __reduce_add_sync(kFull, x0 * static_cast<int>(wr));
                        a2 = __reduce_add_sync(kFull, x0 * static_cast<int>(wc));
                    } else {
                        const int lo = x0 & 0xFF, hi = x0 >> 8;
                        a1 = static_cast<long long>(__reduce_add_sync(kFull, lo * static_cast<int>(wr))) +
                             256ll * __reduce_add_sync(kFull, hi * static_cast<int>(wr));
                        a2 = static_cast<long long>(__reduce_add_sync(kFull, lo * static_cast<int>(wc))) +
                             256ll * __reduce_add_sync(kFull, hi * static_cast<int>(wc));
                    }
                    if (lane == i) {
                        m0 = a0;
                        m1 = a1;
                        m2 = a2;
                    }
                }
                const int sc = seg * 32 + lane;
                if (m1)
                    atomicAdd(s_acc + sc, static_cast<unsigned long long>(m1));
                if (m2)
                    atomicAdd(s_acc + kScans + sc, static_cast<unsigned long long>(m2));
                if (m0)
                    atomicAdd(s_acc + 2 * kScans + sc, static_cast<unsigned long long>(m0));
            }
            if (runs) {
                // one event per iteration (see decode_task): jump the zero-bit run,
                // then the landing slot's step; its nonzero counts scatter
                // (the next event's entry is read before this event's additions,
                // as in the masked sum)
                const uint32_t rt_sa = static_cast<uint32_t>(__cvta_generic_to_shared(s_dec + S.model * kStates));
                int j = 0;
                bool bad = false;
                uint32_t t = tab_load_ordered(S.x, rt_sa);
                while (j < kPairs) {
                    j += static_cast<int>((t >> 14) & 63u);
                    if (j >= kPairs) {
                        bad = j > kPairs;
                        S.x = (t >> 28) & 1u;
                        break;
                    }
                    if (S.bt.n < 10)
                        S.bt.refill();
                    S.x = (t & 1023u) | S.bt.get(static_cast<int>((t >> 10) & 15u));
                    const uint32_t tn = tab_load_ordered(S.x, rt_sa);
                    const long long a = (t >> 20) & 15u, c = (t >> 24) & 15u;
                    if (a) {
                        atomicAdd(s_acc + 2 * j, static_cast<unsigned long long>(a * wr));
                        atomicAdd(s_acc + kScans + 2 * j, static_cast<unsigned long long>(a * wc));
                        atomicAdd(s_acc + 2 * kScans + 2 * j, static_cast<unsigned long long>(a));
                    }
                    if (c) {
                        atomicAdd(s_acc + 2 * j + 1, static_cast<unsigned long long>(c * wr));
                        atomicAdd(s_acc + kScans + 2 * j + 1, static_cast<unsigned long long>(c * wc));
                        atomicAdd(s_acc + 2 * kScans + 2 * j + 1, static_cast<unsigned long long>(c));
                    }
                    ++j;
                    t = tn;
                }
                if (bad)
                    report(st, kErrState);
                else
                    close_paired(S, st);
            } else if (S.form == kPaired) {
                if (over > (W == 1 ? 0xFFu : 0xFFFFu))
                    report(st, kErrValue);
                close_paired(S, st);
            } else if (S.form == kSparse) {
                int prev = -1;
                bool bad = false;
                for (uint32_t k = 0; k < S.c; ++k) {
                    if (S.bt.n < 9)
                        S.bt.refill();
                    const int pos = static_cast<int>(S.bt.get(9));
                    if (S.br.n < 16)
                        S.br.refill();
                    const long long val = S.br.get(8 * W);
                    if (pos <= prev || val == 0) {
                        bad = true;
                        break;
                    }
                    prev = pos;
                    atomicAdd(s_acc + pos, static_cast<unsigned long long>(val * wr));
                    atomicAdd(s_acc + kScans + pos, static_cast<unsigned long long>(val * wc));
                    atomicAdd(s_acc + 2 * kScans + pos, static_cast<unsigned long long>(val));
                }
                if (bad) {
                    report(st, kErrSparse);
                } else {
                    const int pad = static_cast<int>(((9u * S.c + 7u) / 8u) * 8u - 9u * S.c);
                    if (pad) {
                        if (S.bt.n < pad)
                            S.bt.refill();
                        if (S.bt.get(pad) != 0u)
                            report(st, kErrPad);
                    }
                }
            }
        }
        __syncthreads();
        for (int i = threadIdx.x; i < 3 * kScans; i += blockDim.x) {
            out[(static_cast<long long>(i / kScans) * rows + row) * kScans + (i % kScans)] =
                static_cast<long long>(s_acc[i]);
            s_acc[i] = 0ull;
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// a7: block decode into native frames
// ---------------------------------------------------------------------------
// One thread per stream of nblk blocks from `first`: the thread decodes its
// stream's 512 counts in order and stores them down its pixel column of the
// [n * 512][P] frames (neighbouring threads hold neighbouring pixels, so each
// scan's stores are coalesced).  Invalid pixels come out 0.
constexpr int kBlockDecodeThreads = 768;   // 80 registers per thread: the decode loops without spills

template <int W>
__global__ void __launch_bounds__(kBlockDecodeThreads, 1) k_decode_blocks(View v, const uint32_t *__restrict__ dec_g,
                                                          const uint32_t *__restrict__ runs_g, uint32_t skip_models,
                                                          int skip_count, long long first, long long nblk,
                                                          void *__restrict__ out, DevStatus *__restrict__ st)
{
    using T = typename std::conditional<W == 1, uint8_t, uint16_t>::type;
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t *s_dec = smem;
    // the run-event tables of the low-dose models, then the other decode tables
    for (int i = threadIdx.x; i < kModels * kStates / 4; i += blockDim.x)
        reinterpret_cast<uint4 *>(s_dec)[i] = i < skip_count * kStates / 4
                                                  ? __ldg(reinterpret_cast<const uint4 *>(runs_g) + i)
                                                  : __ldg(reinterpret_cast<const uint4 *>(dec_g) + i);
    __syncthreads();
    T *o = reinterpret_cast<T *>(out);
    const long long total = nblk * v.P;
    for (long long sid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; sid < total;
         sid += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long bi = sid / v.P;
        const int p = static_cast<int>(sid - bi * v.P);
        const long long b = first + bi;
        T *dst = o + static_cast<size_t>(bi) * kScans * v.P + p;
        const size_t P = static_cast<size_t>(v.P);
        Stream S;
        S.form = kEmpty;
        S.model = 0;
        S.shift = 0;
        S.base = 0;
        S.c = 0;
        S.x = 0;
        S.x2 = 0;
        S.two = false;
        S.len = 0;
        bool ok = v.valid[p] != 0;
        if (ok)
            ok = locate(v, b, p, S.s, S.len, st);
        if (ok)
            ok = open_stream(S, W, st);
        if (!ok)
            S.form = kEmpty;
        const bool run_model = (skip_models >> S.model) & 1u;
        if (S.form == kPaired && run_model && S.shift == 0 && S.base == 0u) {
            // a low-dose stream: zeros down the column, then its run events (as
            // in the masked sum: jump the zero-bit (0,0) steps, take the step at
            // the slot reached) store its nonzero counts
            for (int i = 0; i < kScans; ++i)
                dst[i * P] = 0;
            const uint32_t rt_sa = static_cast<uint32_t>(__cvta_generic_to_shared(s_dec + S.model * kStates));
            int j = 0;
            bool bad = false;
            while (j < kPairs) {
                const uint32_t t = tab_load(S.x, rt_sa);
                j += static_cast<int>((t >> 14) & 63u);
                if (j >= kPairs) {
                    bad = j > kPairs;
                    S.x = (t >> 28) & 1u;
                    break;
                }
                if (S.bt.n < 10)
                    S.bt.refill();
                S.x = (t & 1023u) | S.bt.get(static_cast<int>((t >> 10) & 15u));
                const uint32_t a = (t >> 20) & 15u, c = (t >> 24) & 15u;
                if (a)
                    dst[static_cast<size_t>(2 * j) * P] = static_cast<T>(a);
                if (c)
                    dst[static_cast<size_t>(2 * j + 1) * P] = static_cast<T>(c);
                ++j;
            }
            if (bad)
                report(st, kErrState);
            else
                close_paired(S, st);
        } else if (S.form == kPaired && S.two && S.shift == 0 && S.base == 0u) {
            // a two-state stream without base or raw bits (models 8-31, whose
            // decode tables are in shared memory): both states' table steps
            // interleaved as in the masked sum, the counts stored as they come
            const uint32_t dec_sa = static_cast<uint32_t>(__cvta_generic_to_shared(s_dec + S.model * kStates));
            for (int seg = 0; seg < 16; ++seg) {
                uint32_t pk[16];
#pragma unroll
                for (int jj = 0; jj < 16; jj += 2) {
                    const uint32_t ea = tab_load(S.x, dec_sa);
                    const uint32_t eb = tab_load(S.x2, dec_sa);
                    if (jj % 3 == 0 && S.bt.n < 30)
                        S.bt.refill();
                    pk[jj] = consume(ea, S.x, S.bt.lo, S.bt.hi, S.bt.n);
                    if ((jj + 1) % 3 == 0 && S.bt.n < 30)
                        S.bt.refill();
                    pk[jj + 1] = consume(eb, S.x2, S.bt.lo, S.bt.hi, S.bt.n);
                }
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    dst[static_cast<size_t>(seg * 32 + 2 * jj) * P] = static_cast<T>(pk[jj] & 0xFFFFu);
                    dst[static_cast<size_t>(seg * 32 + 2 * jj + 1) * P] = static_cast<T>(pk[jj] >> 16);
                }
            }
            close_paired(S, st);
        } else if (S.form == kPaired) {
            // the run-decoded models' decode tables stay in global memory
            const uint32_t *dec = (run_model ? dec_g : s_dec) + S.model * kStates;
            uint32_t over = 0;
            for (int seg = 0; seg < 16; ++seg) {
                uint32_t vv[32];
                paired_segment(S, dec, vv, over);
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    dst[(seg * 32 + i) * P] = static_cast<T>(vv[i]);
            }
            if (over > (W == 1 ? 0xFFu : 0xFFFFu))
                report(st, kErrValue);
            close_paired(S, st);
        } else if (S.form == kLiteral) {
            for (int i = 0; i < kScans; ++i) {
                if (S.bt.n < 16)
                    S.bt.refill();
                dst[i * P] = static_cast<T>(S.bt.get(8 * W));
            }
        } else if (S.form == kSparse) {
            int prev = -1;
            bool bad = false;
            for (uint32_t k = 0; k < S.c; ++k) {
                if (S.bt.n < 9)
                    S.bt.refill();
                const int pos = static_cast<int>(S.bt.get(9));
                if (S.br.n < 16)
                    S.br.refill();
                const uint32_t val = S.br.get(8 * W);
                if (pos <= prev || val == 0u) {
                    bad = true;
                    break;
                }
                for (int i = prev + 1; i < pos; ++i)
                    dst[i * P] = 0;
                dst[pos * P] = static_cast<T>(val);
                prev = pos;
            }
            for (int i = prev + 1; i < kScans; ++i)
                dst[i * P] = 0;
            if (bad) {
                report(st, kErrSparse);
            } else {
                const int pad = static_cast<int>(((9u * S.c + 7u) / 8u) * 8u - 9u * S.c);
                if (pad) {
                    if (S.bt.n < pad)
                        S.bt.refill();
                    if (S.bt.get(pad) != 0u)
                        report(st, kErrPad);
                }
            }
        } else {
            const T c = static_cast<T>(S.form == kConstant ? S.c : 0u);
            for (int i = 0; i < kScans; ++i)
                dst[i * P] = c;
        }
    }
}

// ---------------------------------------------------------------------------
// a7b: scan-range decode (frames)
// ---------------------------------------------------------------------------
// Scans [first, first + n) in native frames: one thread per stream of every
// block the range touches; a stream is decoded only up to the last pair the
// range needs and its counts inside the range are stored down its pixel
// column of out[n][P] (coalesced per scan, as in the block decode).  Literal
// counts are read directly at their byte offset.  Because paired streams
// stop early, their end-of-stream state is not checked here (block decodes
// and queries check it); everything that is read is checked (header, fields,
// form lengths, sparse order, value range, and that no read passes the
// stream's extent).  Invalid pixels come out 0.
template <int W>
__global__ void __launch_bounds__(256) k_decode_range(View v, const uint32_t *__restrict__ dec_g,
                                                     const uint32_t *__restrict__ runs_g, uint32_t skip_models,
                                                     int skip_count, long long first, long long n,
                                                     void *__restrict__ out, DevStatus *__restrict__ st)
{
    using T = typename std::conditional<W == 1, uint8_t, uint16_t>::type;
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t *s_dec = smem;
    __shared__ __align__(8) uint64_t s_bar;
    if (threadIdx.x == 0)
        tables_start(&s_bar, s_dec, dec_g, runs_g, skip_count);
    __syncthreads();
    bool ready = false;
    T *o = reinterpret_cast<T *>(out);
    const long long b0 = first / kScans, b1 = (first + n - 1) / kScans;
    const long long total = (b1 - b0 + 1) * v.P;
    const size_t P = static_cast<size_t>(v.P);
    for (long long sid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; sid < total;
         sid += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long bi = sid / v.P;
        const int p = static_cast<int>(sid - bi * v.P);
        const long long b = b0 + bi;
        // this block's scans inside the range: [lo, hi) of its 512
        const int lo = static_cast<int>(max(first, b * kScans) - b * kScans);
        const int hi = static_cast<int>(min(first + n, (b + 1) * kScans) - b * kScans);
        T *dst = o + (static_cast<size_t>(b * kScans + lo - first)) * P + p;   // row of scan lo
        Stream S;
        S.form = kEmpty;
        S.model = 0;
        S.shift = 0;
        S.base = 0;
        S.c = 0;
        S.x = 0;
        S.x2 = 0;
        S.two = false;
        S.len = 0;
        bool ok = v.valid[p] != 0;
        if (ok)
            ok = locate(v, b, p, S.s, S.len, st);
        if (ok)
            ok = open_stream(S, W, st);
        if (!ok)
            S.form = kEmpty;
        if (S.form == kPaired) {
            if (!ready) {
                if (!tables_wait(&s_bar, st))
                    S.form = kEmpty;
                ready = true;
            }
        }
        const bool run_model = (skip_models >> S.model) & 1u;
        if (S.form == kPaired && run_model && S.shift == 0 && S.base == 0u) {
            // a low-dose stream: zeros over the range, then its run events (jump
            // the zero-bit (0,0) steps, take the step at the slot reached) up to
            // the last pair the range needs, storing the nonzero counts inside it
            for (int sc = lo; sc < hi; ++sc)
                dst[(sc - lo) * P] = 0;
            const uint32_t rt_sa = static_cast<uint32_t>(__cvta_generic_to_shared(s_dec + S.model * kStates));
            const int j_end = (hi + 1) >> 1;        // pairs [0, j_end) hold the range's scans
            int j = 0;
            while (j < j_end) {
                const uint32_t t = tab_load(S.x, rt_sa);
                j += static_cast<int>((t >> 14) & 63u);
                if (j >= j_end)
                    break;
                if (S.bt.n < 10)
                    S.bt.refill();
                S.x = (t & 1023u) | S.bt.get(static_cast<int>((t >> 10) & 15u));
                const uint32_t a = (t >> 20) & 15u, c = (t >> 24) & 15u;
                if (a && 2 * j >= lo && 2 * j < hi)
                    dst[(2 * j - lo) * P] = static_cast<T>(a);
                if (c && 2 * j + 1 >= lo && 2 * j + 1 < hi)
                    dst[(2 * j + 1 - lo) * P] = static_cast<T>(c);
                ++j;
            }
            if (S.bt.consumed() > 8ll * S.tans_len)
                report(st, kErrLength);
        } else if (S.form == kPaired && S.two && S.shift == 0 && S.base == 0u) {
            // a two-state stream without base or raw bits (models 8-31, tables in
            // shared memory): the interleaved table steps up to the range's end
            const uint32_t dec_sa = static_cast<uint32_t>(__cvta_generic_to_shared(s_dec + S.model * kStates));
            const int last_seg = (hi - 1) >> 5;
            for (int seg = 0; seg <= last_seg; ++seg) {
                uint32_t pk[16];
#pragma unroll
                for (int jj = 0; jj < 16; jj += 2) {
                    const uint32_t ea = tab_load(S.x, dec_sa);
                    const uint32_t eb = tab_load(S.x2, dec_sa);
                    if (jj % 3 == 0 && S.bt.n < 30)
                        S.bt.refill();
                    pk[jj] = consume(ea, S.x, S.bt.lo, S.bt.hi, S.bt.n);
                    if ((jj + 1) % 3 == 0 && S.bt.n < 30)
                        S.bt.refill();
                    pk[jj + 1] = consume(eb, S.x2, S.bt.lo, S.bt.hi, S.bt.n);
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int sc = seg * 32 + i;
                    if (sc >= lo && sc < hi)
                        dst[(sc - lo) * P] = static_cast<T>((i & 1) ? (pk[i >> 1] >> 16) : (pk[i >> 1] & 0xFFFFu));
                }
            }
            if (S.bt.consumed() > 8ll * S.tans_len)
                report(st, kErrLength);
        } else if (S.form == kPaired) {
            // the run-decoded models' decode tables stay in global memory
            const uint32_t *dec = (run_model ? dec_g : s_dec) + S.model * kStates;
            uint32_t over = 0;
            const int last_seg = (hi - 1) >> 5;
            for (int seg = 0; seg <= last_seg; ++seg) {
                uint32_t vv[32];
                paired_segment(S, dec, vv, over);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int sc = seg * 32 + i;
                    if (sc >= lo && sc < hi)
                        dst[(sc - lo) * P] = static_cast<T>(vv[i]);
                }
            }
            if (over > (W == 1 ? 0xFFu : 0xFFFFu))
                report(st, kErrValue);
            if (S.bt.consumed() > 8ll * S.tans_len || S.br.consumed() > 8ll * 64 * S.shift)
                report(st, kErrLength);
        } else if (S.form == kLiteral) {
            for (int sc = lo; sc < hi; ++sc)
                dst[(sc - lo) * P] = static_cast<T>(load_native(S.s + 2 + sc * W, W));
        } else if (S.form == kSparse) {
            for (int sc = lo; sc < hi; ++sc)
                dst[(sc - lo) * P] = 0;
            int prev = -1;
            for (uint32_t k = 0; k < S.c; ++k) {
                if (S.bt.n < 9)
                    S.bt.refill();
                const int pos = static_cast<int>(S.bt.get(9));
                if (S.br.n < 16)
                    S.br.refill();
                const uint32_t val = S.br.get(8 * W);
                if (pos <= prev || val == 0u) {
                    report(st, kErrSparse);
                    break;
                }
                if (pos >= hi)
                    break;
                if (pos >= lo)
                    dst[(pos - lo) * P] = static_cast<T>(val);
                prev = pos;
            }
        } else {
            const T c = static_cast<T>(S.form == kConstant ? S.c : 0u);
            for (int sc = lo; sc < hi; ++sc)
                dst[(sc - lo) * P] = c;
        }
    }
    __syncthreads();
    // a CTA leaves only after its table copy has landed
    if (threadIdx.x == 0)
        tables_wait(&s_bar, st);
}

// float32 square-root amplitude of decoded counts (the feed's second output;
// sqrtf is the correctly rounded square root)
template <typename T>
__global__ void k_amplitude(const T *__restrict__ in, float *__restrict__ out, long long n)
{
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x)
        out[i] = sqrtf(static_cast<float>(in[i]));
}

// SM count of the current device (cached per device).
int sm_count()
{
    static std::mutex mu;
    static std::map<int, int> cache;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(dev);
    if (it != cache.end())
        return it->second;
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0)
        n = 1;
    cache[dev] = n;
    return n;
}

// Raise a kernel's dynamic shared-memory limit to `bytes` on the current
// device (the attribute belongs to each device's context), once.
cudaError_t ensure_smem(const void *fn, size_t bytes)
{
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, size_t> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    std::lock_guard<std::mutex> lk(mu);
    size_t &have = done[std::make_pair(fn, dev)];
    if (have >= bytes)
        return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
    if (e == cudaSuccess)
        have = bytes;
    return e;
}

constexpr size_t kTableBytes = static_cast<size_t>(kModels) * kStates * sizeof(uint32_t);

// ---------------------------------------------------------------------------
// interaction index: build
// ---------------------------------------------------------------------------
// Pass 1: every stream of nblk blocks from block b0 is decoded and its counts
// added per scan into its leaf's sums, leafsum[bb][leaf][512] (global, zeroed
// by the caller).  The list is the polar slot order (64 slots per leaf,
// padding slots hold P); a task is one block and 32 slots (half a leaf).
template <int W>
__global__ void __launch_bounds__(768, 1) k_index_sums(View v, const uint32_t *__restrict__ dec_g,
                                                      const uint32_t *__restrict__ runs_g, uint32_t skip_models,
                                                      int skip_count, const uint32_t *__restrict__ slots, int L,
                                                      long long b0, int nblk, uint32_t *__restrict__ leafsum,
                                                      DevStatus *__restrict__ st)
{
    constexpr int THREADS = 768, MAXW = THREADS / 32;
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t *s_dec = smem;
    uint32_t *s_stage = smem + kModels * kStates;
    __shared__ __align__(8) uint64_t s_bar;
    __shared__ uint32_t s_cnt[2];
    if (threadIdx.x == 0)
        tables_start(&s_bar, s_dec, dec_g, runs_g, skip_count);
    if (threadIdx.x < 2)
        s_cnt[threadIdx.x] = 0u;
    __syncthreads();
    bool ready = false;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long tiles = 2ll * L;
    const long long total = tiles * nblk;
    for (long long t = static_cast<long long>(blockIdx.x) * MAXW + warp; t < total;
         t += static_cast<long long>(gridDim.x) * MAXW) {
        const long long bb = t / tiles;
        const int tile = static_cast<int>(t - bb * tiles);
        decode_task<W, false>(v, s_dec, dec_g, skip_models, slots, static_cast<uint32_t>(64 * L), 0u, tile, b0 + bb,
                              leafsum + (bb * L + tile / 2) * kScans, s_stage + warp * 16, s_cnt, &s_bar, ready,
                              lane, st);
    }
    __syncthreads();
    if (threadIdx.x == 0 && !ready)
        tables_wait(&s_bar, st);
}

// The 512 sums of group g of block bb: a leaf's from leafsum; a root's as
// the sum of its leaves [root_leaf0[r], root_leaf0[r+1]).
__device__ __forceinline__ uint32_t group_sum(const uint32_t *leafsum, const int *root_leaf0, int L, long long bb,
                                              int g, int sc)
{
    if (g < L)
        return leafsum[(bb * L + g) * kScans + sc];
    const int r = g - L;
    uint32_t t = 0;
    for (int l = root_leaf0[r]; l < root_leaf0[r + 1]; ++l)
        t += leafsum[(bb * L + l) * kScans + sc];
    return t;
}

// Pass 2 (one CTA per block): each group's width code from its largest sum,
// then the byte offsets (exclusive scan over the groups) into desc[bb][G];
// the block's total bytes into total[bb].
__global__ void __launch_bounds__(1024) k_index_size(const uint32_t *__restrict__ leafsum,
                                                    const int *__restrict__ root_leaf0, int L, int G,
                                                    uint32_t *__restrict__ desc, unsigned long long *__restrict__ total)
{
    extern __shared__ uint32_t s_sz[];     // [G] bytes of each group
    const long long bb = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int g = warp; g < G; g += nw) {
        uint32_t mx = 0;
        for (int sc = lane; sc < kScans; sc += 32)
            mx = max(mx, group_sum(leafsum, root_leaf0, L, bb, g, sc));
        mx = __reduce_max_sync(kFull, mx);
        if (lane == 0)
            s_sz[g] = mx == 0u ? 0u : (mx <= 0xFFu ? 1u : (mx <= 0xFFFFu ? 2u : 3u));
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long off = 0;
        for (int g = 0; g < G; ++g) {
            const uint32_t code = s_sz[g];
            desc[bb * G + g] = static_cast<uint32_t>(off) | (code << 30);
            off += code == 0u ? 0u : (static_cast<unsigned long long>(kScans) << (code - 1u));
        }
        total[bb] = off;
    }
}

// Pass 3: write each group's sums at its width to base[b0 + bb] + offset.
__global__ void __launch_bounds__(512) k_index_pack(const uint32_t *__restrict__ leafsum,
                                                   const int *__restrict__ root_leaf0, int L, int G, long long b0,
                                                   const uint32_t *__restrict__ desc_all,
                                                   const unsigned long long *__restrict__ base)
{
    const long long bb = blockIdx.y;
    const int g = blockIdx.x;
    const uint32_t d = desc_all[(b0 + bb) * G + g];
    const uint32_t code = d >> 30;
    if (code == 0u)
        return;
    const unsigned long long a = base[b0 + bb] + (d & 0x3FFFFFFFu);
    for (int sc = threadIdx.x; sc < kScans; sc += blockDim.x) {
        const uint32_t val = group_sum(leafsum, root_leaf0, L, bb, g, sc);
        if (code == 1u)
            reinterpret_cast<uint8_t *>(a)[sc] = static_cast<uint8_t>(val);
        else if (code == 2u)
            reinterpret_cast<uint16_t *>(a)[sc] = static_cast<uint16_t>(val);
        else
            reinterpret_cast<uint32_t *>(a)[sc] = val;
    }
}

// ---------------------------------------------------------------------------
// interaction index: plan (one CTA per root, one warp per leaf)
// ---------------------------------------------------------------------------
// A leaf whose every pixel is in the mask (full query), or whose every pixel
// enters, or every pixel leaves, the mask (delta) becomes one index item; a
// root whose leaves all do so in the same direction becomes one root item
// instead.  In a full query, a leaf partly in the mask becomes an item plus
// its unmasked pixels with a minus sign when their decode costs less than
// the masked pixels' (planner weights: a pair-by-pair stream kPlanHeavy, a
// light one kPlanLight, an item kPlanItem).  The remaining masked (changed)
// pixels go to the residual list as in k_plan.  The counts are count[0]
// heavy, count[1] light, count[2] items.  Entries with bit 31 set subtract,
// so the decode that follows is the signed (delta) instantiation.
constexpr uint32_t kPlanHeavy = 16, kPlanLight = 1, kPlanItem = 2;
__global__ void __launch_bounds__(512) k_plan_index(const uint8_t *__restrict__ mask,
                                                   const uint8_t *__restrict__ pclass,
                                                   uint8_t *__restrict__ base_mask, int P, int mode,
                                                   const uint32_t *__restrict__ slots,
                                                   const int *__restrict__ root_leaf0, int R,
                                                   uint32_t *__restrict__ list, uint32_t *__restrict__ items,
                                                   uint32_t *__restrict__ count, uint32_t *__restrict__ count_next,
                                                   uint4 *__restrict__ out, uint4 *__restrict__ keep, long long n_vec)
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (blockIdx.x == 0 && threadIdx.x < 4)
        count_next[threadIdx.x] = 0u;
    if (static_cast<int>(blockIdx.x) < R) {
        constexpr int NW = 16;
        __shared__ int s_state[NW];            // per leaf: 1 all enter/in, 2 all leave, 3 item minus
                                               // unmasked pixels, 0 otherwise, -1 none
        __shared__ uint32_t s_h[NW], s_l[NW], s_at[2];
        const int r = blockIdx.x;
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        const int l0 = root_leaf0[r], nl = root_leaf0[r + 1] - l0;
        const int leaf = l0 + warp;
        bool emit[2] = {false, false}, light[2] = {false, false};
        uint32_t entry[2] = {0u, 0u};
        int state = -1;
        if (warp < nl) {
            bool all_in = true, all_out = true;
            const uint2 pp = reinterpret_cast<const uint2 *>(slots + leaf * 64)[lane];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const uint32_t p = k ? pp.y : pp.x;
                if (p >= static_cast<uint32_t>(P))
                    continue;
                const uint8_t mk = mask[p];
                const bool nw = mk != 0;
                const bool od = base_mask[p] != 0;
                bool add, rem;
                if (mode == 0) {
                    add = nw;
                    rem = false;
                } else {
                    add = nw && !od;
                    rem = !nw && od;
                }
                all_in = all_in && add;
                all_out = all_out && rem;
                emit[k] = add || rem;
                entry[k] = p | (rem ? 0x80000000u : 0u);
                light[k] = pclass[p] != 0;
                base_mask[p] = mk;
            }
            all_in = __all_sync(kFull, all_in);
            all_out = __all_sync(kFull, all_out) && mode == 1;
            state = all_in ? 1 : (all_out ? 2 : 0);
            if (mode == 0) {
                // planner: decode the leaf's masked pixels, or take its stored sums
                // and subtract its unmasked pixels, whichever decodes less (cost of
                // a stream by its class; an item reads 512 stored sums)
                uint32_t c_in = 0, c_out = 0;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const uint32_t p = k ? pp.y : pp.x;
                    const uint32_t c = light[k] ? kPlanLight : kPlanHeavy;
                    if (p < static_cast<uint32_t>(P)) {
                        c_in += emit[k] ? c : 0u;
                        c_out += emit[k] ? 0u : c;
                    }
                }
                c_in = __reduce_add_sync(kFull, c_in);
                c_out = __reduce_add_sync(kFull, c_out);
                if (state == 0 && kPlanItem + c_out < c_in) {
                    state = 3;
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const uint32_t p = k ? pp.y : pp.x;
                        emit[k] = p < static_cast<uint32_t>(P) && !emit[k];
                        entry[k] = p | 0x80000000u;
                    }
                }
            }
        }
        if (lane == 0)
            s_state[warp] = state;
        __syncthreads();
        // the root as one item when all its leaves are wholly in (or wholly leave)
        int rs = s_state[0];
        for (int k = 1; k < nl; ++k)
            rs = s_state[k] == rs ? rs : 0;
        const bool root_item = nl > 0 && (rs == 1 || rs == 2);
        if (state == 1 || state == 2 || root_item) {
            emit[0] = emit[1] = false;        // covered by an index item
        }
        // index items: one reservation per CTA (the root, or its whole leaves in order)
        if (threadIdx.x == 0) {
            if (root_item) {
                items[atomicAdd(count + 2, 1u)] = static_cast<uint32_t>(r) | (1u << 30) | (rs == 2 ? 0x80000000u : 0u);
            } else {
                uint32_t nf = 0;
                for (int k = 0; k < nl; ++k)
                    nf += s_state[k] > 0;
                if (nf) {
                    uint32_t at = atomicAdd(count + 2, nf);
                    for (int k = 0; k < nl; ++k)
                        if (s_state[k] > 0)
                            items[at++] = static_cast<uint32_t>(l0 + k) | (s_state[k] == 2 ? 0x80000000u : 0u);
                }
            }
        }
        // residual pixels: block-level reservations per class, as in k_plan
        uint32_t nh = 0, nlt = 0;
        unsigned bh[2], bl[2];
        for (int k = 0; k < 2; ++k) {
            bh[k] = __ballot_sync(kFull, emit[k] && !light[k]);
            bl[k] = __ballot_sync(kFull, emit[k] && light[k]);
            nh += __popc(bh[k]);
            nlt += __popc(bl[k]);
        }
        if (lane == 0) {
            s_h[warp] = nh;
            s_l[warp] = nlt;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t th = 0, tl = 0;
            for (int w = 0; w < NW; ++w) {
                const uint32_t a = s_h[w], c = s_l[w];
                s_h[w] = th;
                s_l[w] = tl;
                th += a;
                tl += c;
            }
            s_at[0] = th ? atomicAdd(count, th) : 0u;
            s_at[1] = tl ? atomicAdd(count + 1, tl) : 0u;
        }
        __syncthreads();
        const unsigned below = (1u << lane) - 1u;
        uint32_t oh = s_at[0] + s_h[warp], ol = s_at[1] + s_l[warp];
        for (int k = 0; k < 2; ++k) {
            if (emit[k] && !light[k])
                list[oh + __popc(bh[k] & below)] = entry[k];
            if (emit[k] && light[k])
                list[P - 1 - (ol + __popc(bl[k] & below))] = entry[k];
            oh += __popc(bh[k]);
            ol += __popc(bl[k]);
        }
        return;
    }
    const long long stride = static_cast<long long>(gridDim.x - R) * blockDim.x;
    for (long long i = static_cast<long long>(blockIdx.x - R) * blockDim.x + threadIdx.x; i < n_vec; i += stride) {
        if (mode == 0) {
            out[i] = make_uint4(0u, 0u, 0u, 0u);
            keep[i] = make_uint4(0u, 0u, 0u, 0u);
        } else {
            out[i] = keep[i];
        }
    }
}

}  // namespace

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
cudaError_t launch_generate(void *out, int bits, uint64_t seed, int64_t scan0, int64_t n_scans, int P,
                            const uint32_t *pclass, const uint32_t *desc, const uint64_t *thr, cudaStream_t st)
{
    if (n_scans <= 0 || P <= 0)
        return cudaSuccess;
    dim3 block(256);
    dim3 grid((P + 255) / 256, static_cast<unsigned>(n_scans < 4096 ? n_scans : 4096));
    const uint4 *d = reinterpret_cast<const uint4 *>(desc);
    if (bits == 8)
        k_generate<uint8_t><<<grid, block, 0, st>>>(static_cast<uint8_t *>(out), seed, scan0, n_scans, P, pclass,
                                                    d, thr, 0xFFu);
    else
        k_generate<uint16_t><<<grid, block, 0, st>>>(static_cast<uint16_t *>(out), seed, scan0, n_scans, P,
                                                     pclass, d, thr, 0xFFFFu);
    return cudaGetLastError();
}

cudaError_t launch_enc_streams(const void *counts, int w, int P, int nblk, Tables tb, uint4 *desc, uint32_t *slots,
                               unsigned long long *stats, uint8_t *pclass, cudaStream_t st)
{
    const long long total = static_cast<long long>(nblk) * P;
    const unsigned grid = static_cast<unsigned>((total + kEncThreads - 1) / kEncThreads);
    if (w == 1)
        k_enc_streams<uint8_t><<<grid, kEncThreads, 0, st>>>(static_cast<const uint8_t *>(counts), P, nblk, tb,
                                                             desc, slots, stats, pclass);
    else
        k_enc_streams<uint16_t><<<grid, kEncThreads, 0, st>>>(static_cast<const uint16_t *>(counts), P, nblk, tb,
                                                              desc, slots, stats, pclass);
    return cudaGetLastError();
}

cudaError_t launch_enc_layout(uint4 *desc, int P, int G, int nblk, uint32_t *groups, uint32_t *blk_len,
                              cudaStream_t st)
{
    k_enc_layout<<<nblk, kLayoutThreads, 0, st>>>(desc, P, G, groups, blk_len);
    return cudaGetLastError();
}

cudaError_t launch_enc_compact(const void *counts, int w, int P, int nblk, const uint4 *desc,
                               const uint32_t *slots, const unsigned long long *blk_dst, cudaStream_t st)
{
    const dim3 grid((P + kCompactThreads - 1) / kCompactThreads, nblk);
    const int smem = kCompactBytes + 32;
    cudaError_t e = w == 1 ? ensure_smem(reinterpret_cast<const void *>(k_enc_compact<uint8_t>), smem)
                           : ensure_smem(reinterpret_cast<const void *>(k_enc_compact<uint16_t>), smem);
    if (e != cudaSuccess)
        return e;
    if (w == 1)
        k_enc_compact<uint8_t><<<grid, kCompactThreads, smem, st>>>(static_cast<const uint8_t *>(counts), P, nblk,
                                                                     desc, slots, blk_dst);
    else
        k_enc_compact<uint16_t><<<grid, kCompactThreads, smem, st>>>(static_cast<const uint16_t *>(counts), P, nblk,
                                                                      desc, slots, blk_dst);
    return cudaGetLastError();
}

cudaError_t launch_plan(const uint8_t *mask, const uint8_t *valid, const uint8_t *pclass, uint8_t *base_mask,
                        int P, int mode, uint32_t *list, uint32_t *count, uint32_t *count_next, void *out,
                        void *keep, long long n_elems, int out_bytes, cudaStream_t st,
                        const unsigned long long *total, int stride)
{
    const long long n_vec = n_elems * out_bytes / 16;
    const int n_list = (P + kPlanThreads - 1) / kPlanThreads;
    int fill = static_cast<int>((n_vec + kPlanThreads * 4 - 1) / (kPlanThreads * 4));
    fill = fill < 1 ? 1 : (fill > 8 * sm_count() ? 8 * sm_count() : fill);
    k_plan<<<n_list + fill, kPlanThreads, 0, st>>>(mask, valid, pclass, base_mask, P, mode, n_list, list, count,
                                                   count_next, static_cast<uint4 *>(out), static_cast<uint4 *>(keep),
                                                   n_vec, total, stride, out_bytes);
    return cudaGetLastError();
}

template <int W, int TH, bool DELTA>
cudaError_t launch_dr(View v, Tables tb, const uint32_t *list, const uint32_t *count, int stride, long long rows,
                      void *out, void *keep, int out_bytes, IndexView ix, DevStatus *status, int n_sm,
                      cudaStream_t st)
{
    // the run-decoded models are a prefix 0..k-1 (their (0,0) share falls as lambda grows)
    const int skip_count = __builtin_popcount(tb.skip_models);
    const size_t smem = kTableBytes +
                        static_cast<size_t>(TH / 32) * 16 * sizeof(uint32_t) +
                        static_cast<size_t>(kMaxSlots) * kScans * sizeof(uint32_t);
    const cudaError_t e = ensure_smem(reinterpret_cast<const void *>(k_decode_reduce<W, TH, DELTA>), smem);
    if (e != cudaSuccess)
        return e;
    // programmatic dependent launch: the CTAs may become resident and load their
    // tables while the preceding kernel (the plan) is still running
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n_sm);
    cfg.blockDim = dim3(TH);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_decode_reduce<W, TH, DELTA>, v, tb.dec, tb.runs, tb.skip_models, skip_count,
                              list, count, stride, rows, out, keep, out_bytes, ix, status);
}

cudaError_t preload_query_kernels()
{
    const void *fns[] = {reinterpret_cast<const void *>(k_decode_reduce<1, 768, false>),
                         reinterpret_cast<const void *>(k_decode_reduce<2, 512, false>)};
    const size_t smem[] = {kTableBytes + 768 / 32 * 16 * sizeof(uint32_t) + kMaxSlots * kScans * sizeof(uint32_t),
                           kTableBytes + 512 / 32 * 16 * sizeof(uint32_t) + kMaxSlots * kScans * sizeof(uint32_t)};
    for (int i = 0; i < 2; ++i) {
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, fns[i]);
        if (e == cudaSuccess)
            e = ensure_smem(fns[i], smem[i]);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

cudaError_t launch_decode_reduce(View v, Tables tb, const uint32_t *list, const uint32_t *count, int stride,
                                 long long rows, void *out, int out_bytes, DevStatus *status, int n_sm,
                                 cudaStream_t st, bool delta, void *keep, IndexView ix, bool signed_list)
{
    // u8 deltas (few tasks, each warp's decode latency is the critical path)
    // run at 512 threads, with room for more registers; full queries at 768,
    // or 640 when their list has subtracted entries (index plans, complement):
    // the signed decode needs a few more registers than 768 threads leave
    if (v.w == 1) {
        if (delta)
            return launch_dr<1, 512, true>(v, tb, list, count, stride, rows, out, keep, out_bytes, ix, status, n_sm,
                                           st);
        if (signed_list)
            return launch_dr<1, 640, true>(v, tb, list, count, stride, rows, out, keep, out_bytes, ix, status, n_sm,
                                           st);
        return launch_dr<1, 768, false>(v, tb, list, count, stride, rows, out, keep, out_bytes, ix, status, n_sm, st);
    }
    return (delta || signed_list)
               ? launch_dr<2, 512, true>(v, tb, list, count, stride, rows, out, keep, out_bytes, ix, status, n_sm, st)
               : launch_dr<2, 512, false>(v, tb, list, count, stride, rows, out, keep, out_bytes, ix, status, n_sm,
                                          st);
}

cudaError_t launch_decode_blocks(View v, Tables tb, long long first, long long n, void *out, DevStatus *status,
                                 cudaStream_t st)
{
    const size_t smem = kTableBytes;
    const int grid = sm_count();
    const cudaError_t e = v.w == 1 ? ensure_smem(reinterpret_cast<const void *>(k_decode_blocks<1>), smem)
                                   : ensure_smem(reinterpret_cast<const void *>(k_decode_blocks<2>), smem);
    if (e != cudaSuccess)
        return e;
    const int skip_count = __builtin_popcount(tb.skip_models);
    if (v.w == 1)
        k_decode_blocks<1><<<grid, kBlockDecodeThreads, smem, st>>>(v, tb.dec, tb.runs, tb.skip_models, skip_count,
                                                                    first, n, out, status);
    else
        k_decode_blocks<2><<<grid, kBlockDecodeThreads, smem, st>>>(v, tb.dec, tb.runs, tb.skip_models, skip_count,
                                                                    first, n, out, status);
    return cudaGetLastError();
}

cudaError_t launch_decode_range(View v, Tables tb, long long first, long long n, void *out, DevStatus *status,
                                cudaStream_t st)
{
    const int skip_count = __builtin_popcount(tb.skip_models);
    const size_t smem = kTableBytes;
    const cudaError_t e = v.w == 1 ? ensure_smem(reinterpret_cast<const void *>(k_decode_range<1>), smem)
                                   : ensure_smem(reinterpret_cast<const void *>(k_decode_range<2>), smem);
    if (e != cudaSuccess)
        return e;
    const long long blocks = (first + n - 1) / kScans - first / kScans + 1;
    long long grid = (blocks * v.P + 255) / 256;
    grid = grid < 1 ? 1 : (grid > 4ll * sm_count() ? 4ll * sm_count() : grid);
    if (v.w == 1)
        k_decode_range<1><<<static_cast<int>(grid), 256, smem, st>>>(v, tb.dec, tb.runs, tb.skip_models, skip_count,
                                                                      first, n, out, status);
    else
        k_decode_range<2><<<static_cast<int>(grid), 256, smem, st>>>(v, tb.dec, tb.runs, tb.skip_models, skip_count,
                                                                      first, n, out, status);
    return cudaGetLastError();
}

cudaError_t launch_moments(View v, Tables tb, const uint32_t *list, const uint32_t *count, const int32_t *weights,
                           int stride, long long rows, long long *out, DevStatus *status, cudaStream_t st)
{
    const size_t smem = kTableBytes + 3 * kScans * sizeof(unsigned long long);
    const int skip_count = __builtin_popcount(tb.skip_models);
    const cudaError_t e = v.w == 1 ? ensure_smem(reinterpret_cast<const void *>(k_moments<1>), smem)
                                   : ensure_smem(reinterpret_cast<const void *>(k_moments<2>), smem);
    if (e != cudaSuccess)
        return e;
    long long grid = rows < 1 ? 1 : rows;
    grid = grid > sm_count() ? sm_count() : grid;
    if (v.w == 1)
        k_moments<1><<<static_cast<int>(grid), 512, smem, st>>>(v, tb.dec, tb.runs, tb.skip_models, skip_count, list,
                                                                 count, weights, stride, rows, out, status);
    else
        k_moments<2><<<static_cast<int>(grid), 512, smem, st>>>(v, tb.dec, tb.runs, tb.skip_models, skip_count, list,
                                                                 count, weights, stride, rows, out, status);
    return cudaGetLastError();
}

cudaError_t launch_amplitude(const void *counts, int w, float *amp, long long n, cudaStream_t st)
{
    long long grid = (n + 255) / 256;
    grid = grid < 1 ? 1 : (grid > 16ll * sm_count() ? 16ll * sm_count() : grid);
    if (w == 1)
        k_amplitude<uint8_t><<<static_cast<int>(grid), 256, 0, st>>>(static_cast<const uint8_t *>(counts), amp, n);
    else
        k_amplitude<uint16_t><<<static_cast<int>(grid), 256, 0, st>>>(static_cast<const uint16_t *>(counts), amp, n);
    return cudaGetLastError();
}

cudaError_t launch_index_sums(View v, Tables tb, const uint32_t *slots, int L, long long b0, int nblk,
                              uint32_t *leafsum, DevStatus *status, int n_sm, cudaStream_t st)
{
    const int skip_count = __builtin_popcount(tb.skip_models);
    const size_t smem = kTableBytes + 24 * 16 * sizeof(uint32_t);
    const cudaError_t e = v.w == 1 ? ensure_smem(reinterpret_cast<const void *>(k_index_sums<1>), smem)
                                   : ensure_smem(reinterpret_cast<const void *>(k_index_sums<2>), smem);
    if (e != cudaSuccess)
        return e;
    if (v.w == 1)
        k_index_sums<1><<<n_sm, 768, smem, st>>>(v, tb.dec, tb.runs, tb.skip_models, skip_count,
                                                  slots, L, b0, nblk, leafsum, status);
    else
        k_index_sums<2><<<n_sm, 768, smem, st>>>(v, tb.dec, tb.runs, tb.skip_models, skip_count,
                                                  slots, L, b0, nblk, leafsum, status);
    return cudaGetLastError();
}

cudaError_t launch_index_size(const uint32_t *leafsum, const int *root_leaf0, int L, int G, int nblk, uint32_t *desc,
                              unsigned long long *total, cudaStream_t st)
{
    k_index_size<<<nblk, 1024, static_cast<size_t>(G) * 4, st>>>(leafsum, root_leaf0, L, G, desc, total);
    return cudaGetLastError();
}

cudaError_t launch_index_pack(const uint32_t *leafsum, const int *root_leaf0, int L, int G, long long b0, int nblk,
                              const uint32_t *desc_all, const unsigned long long *base, cudaStream_t st)
{
    k_index_pack<<<dim3(G, nblk), 512, 0, st>>>(leafsum, root_leaf0, L, G, b0, desc_all, base);
    return cudaGetLastError();
}

cudaError_t launch_plan_index(const uint8_t *mask, const uint8_t *pclass, uint8_t *base_mask, int P, int mode,
                              const uint32_t *slots, const int *root_leaf0, int R, uint32_t *list, uint32_t *items,
                              uint32_t *count, uint32_t *count_next, void *out, void *keep, long long n_elems,
                              int out_bytes, cudaStream_t st)
{
    const long long n_vec = n_elems * out_bytes / 16;
    int fill = static_cast<int>((n_vec + 512 * 4 - 1) / (512 * 4));
    fill = fill < 1 ? 1 : (fill > 4 * sm_count() ? 4 * sm_count() : fill);
    k_plan_index<<<R + fill, 512, 0, st>>>(mask, pclass, base_mask, P, mode, slots, root_leaf0, R, list, items,
                                           count, count_next, static_cast<uint4 *>(out), static_cast<uint4 *>(keep),
                                           n_vec);
    return cudaGetLastError();
}

}  // namespace qem
