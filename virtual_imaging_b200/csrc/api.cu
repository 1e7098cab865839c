// api.cu -- C ABI of libqem: the resident, its arenas, query planning on the
// host side, per-stride baselines and the deferred error status.
//
// Page "Paired-count resident layout": "Operation pipeline" steps 1-6 and
// "Contract" (virtual image dtype rule, malformed streams raise, queued
// queries with a failed decode invalidating the incremental plan).
#include <algorithm>
#include <chrono>
#include <cmath>
#include <cstring>
#include <map>
#include <numeric>
#include <thread>
#include <vector>

#include "qem_internal.h"

using namespace qem;

namespace {

constexpr size_t kArenaMax = size_t(1) << 30;       // payload allocation unit
constexpr size_t kBatchRawBytes = size_t(512) << 20; // raw counts encoded per batch (one host
                                                      // synchronisation each, for the block placement)
constexpr double kWaitSeconds = 60.0;

enum BaseState { kNone = 0, kValid = 1, kTainted = 2 };

struct Baseline {
    uint8_t *d_mask = nullptr;
    void *d_img = nullptr;
    int out_bits = 0;
    int state = kNone;
    bool pending = false;     // written since the last successful finish
};

struct Arena {
    uint8_t *p = nullptr;
    size_t cap = 0;
    size_t used = 0;
};

struct ProfEvent {
    int kernel;
    cudaEvent_t a, b;
};

}  // namespace

struct qem_resident {
    int device = 0;
    int64_t scan_rows = 0, scan_cols = 0;
    int det_rows = 0, det_cols = 0;
    int bits = 8, w = 1;
    int P = 0, G = 0;
    int64_t B = 0, B_done = 0;
    int n_valid = 0;
    int out_bits_auto = 32;
    int n_sm = 1;

    uint8_t *d_valid = nullptr;
    uint8_t *d_pclass = nullptr;                // per pixel: 1 = light streams (from block 0)
    uint32_t *d_groups = nullptr;
    unsigned long long *d_blk_ptr = nullptr;
    uint32_t *d_blk_len = nullptr;
    std::vector<uint64_t> blk_len;
    std::vector<unsigned long long> blk_ptr;
    std::vector<Arena> arenas;

    uint32_t *d_dec = nullptr, *d_enc_sym = nullptr, *d_cost = nullptr, *d_amax = nullptr;
    uint32_t *d_runs = nullptr;
    uint32_t skip_models = 0;
    uint16_t *d_enc_slot = nullptr;

    uint4 *d_desc = nullptr;
    uint32_t *d_slots = nullptr;
    size_t scratch_streams = 0;
    unsigned long long *d_stats = nullptr;
    uint32_t *h_len = nullptr;                  // pinned
    unsigned long long *h_ptr = nullptr;        // pinned
    size_t pinned_blocks = 0;

    uint32_t *d_list = nullptr;
    uint32_t *d_count = nullptr;                // two sets of (heavy, light, items, -) counters, used in turn
    int count_pair = 0;                         // the set the next query fills
    std::vector<uint8_t> h_valid;

    // interaction index (page "Operation pipeline" step 3)
    bool has_index = false;
    int idx_L = 0, idx_R = 0;
    double idx_center[2] = {0.0, 0.0};
    uint32_t *d_idx_slots = nullptr;            // [64 L] pixel of each polar slot (P = padding)
    int *d_idx_root_leaf0 = nullptr;            // [R + 1]
    uint32_t *d_idx_desc = nullptr;             // [B][L + R]
    unsigned long long *d_idx_base = nullptr;   // [B]
    uint32_t *d_idx_items = nullptr;            // [L + R] items of the current query
    std::vector<Arena> idx_arenas;
    uint64_t idx_bytes = 0;
    uint8_t *d_mom_mask = nullptr;              // scratch mask store of the moments plan
    unsigned long long *d_total = nullptr;      // cached full-detector image [B][512] (complement queries)
    uint8_t *d_tot_mask = nullptr;              // scratch mask store of its plan
    bool total_ready = false;
    void *noalloc_scratch = nullptr;            // allocation-free masked sum: fixed working array
    uint32_t *noalloc_flags = nullptr;          // and its pinned status word (owned by noalloc.cu)
    DevStatus *d_status = nullptr;
    DevStatus *h_status = nullptr;              // pinned
    std::map<int, Baseline> baselines;

    uint64_t form_count[5] = {0, 0, 0, 0, 0};
    uint64_t model_count[32] = {0};

    bool prof = false;
    std::vector<ProfEvent> events;
    qem_profile_t prof_acc{};

    Tables tables() const { return Tables{d_dec, d_enc_sym, d_enc_slot, d_cost, d_amax, d_runs, skip_models}; }
    View view() const { return View{d_groups, d_blk_ptr, d_blk_len, d_valid, P, G, w, B}; }
};

namespace {

int cuda_status(cudaError_t e)
{
    if (e == cudaSuccess)
        return QEM_OK;
    return e == cudaErrorMemoryAllocation ? QEM_ERR_OOM : QEM_ERR_CUDA;
}

#define QEM_CK(expr)                                   \
    do {                                               \
        const cudaError_t qem_e_ = (expr);             \
        if (qem_e_ != cudaSuccess)                     \
            return cuda_status(qem_e_);                \
    } while (0)

template <typename F>
int timed(qem_resident *r, int kernel, cudaStream_t st, F &&launch)
{
    if (!r->prof)
        return cuda_status(launch());
    ProfEvent ev{kernel, nullptr, nullptr};
    QEM_CK(cudaEventCreate(&ev.a));
    QEM_CK(cudaEventCreate(&ev.b));
    QEM_CK(cudaEventRecord(ev.a, st));
    const cudaError_t e = launch();
    QEM_CK(cudaEventRecord(ev.b, st));
    r->events.push_back(ev);
    return cuda_status(e);
}

// Wait for everything queued on `st` so far, with a time limit.
int bounded_wait(cudaStream_t st)
{
    cudaEvent_t ev;
    QEM_CK(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
    cudaError_t e = cudaEventRecord(ev, st);
    if (e != cudaSuccess) {
        cudaEventDestroy(ev);
        return cuda_status(e);
    }
    const auto t0 = std::chrono::steady_clock::now();
    int rc = QEM_OK;
    for (;;) {
        e = cudaEventQuery(ev);
        if (e == cudaSuccess)
            break;
        if (e != cudaErrorNotReady) {
            rc = cuda_status(e);
            break;
        }
        const double dt = std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
        if (dt > kWaitSeconds) {
            rc = QEM_ERR_TIMEOUT;
            break;
        }
        std::this_thread::sleep_for(std::chrono::microseconds(dt < 0.01 ? 2 : 200));
    }
    cudaEventDestroy(ev);
    return rc;
}

template <typename T>
int dalloc(T **p, size_t bytes)
{
    void *q = nullptr;
    QEM_CK(cudaMalloc(&q, bytes ? bytes : 16));
    *p = static_cast<T *>(q);
    return QEM_OK;
}

void release(qem_resident *r)
{
    for (auto &ev : r->events) {
        cudaEventDestroy(ev.a);
        cudaEventDestroy(ev.b);
    }
    for (auto &a : r->arenas)
        cudaFree(a.p);
    for (auto &a : r->idx_arenas)
        cudaFree(a.p);
    cudaFree(r->d_idx_slots);
    cudaFree(r->d_idx_root_leaf0);
    cudaFree(r->d_idx_desc);
    cudaFree(r->d_idx_base);
    cudaFree(r->d_idx_items);
    cudaFree(r->d_mom_mask);
    cudaFree(r->d_total);
    cudaFree(r->d_tot_mask);
    for (auto &kv : r->baselines) {
        cudaFree(kv.second.d_mask);
        cudaFree(kv.second.d_img);
    }
    cudaFree(r->d_valid);
    cudaFree(r->d_pclass);
    cudaFree(r->d_groups);
    cudaFree(r->d_blk_ptr);
    cudaFree(r->d_blk_len);
    cudaFree(r->d_dec);
    cudaFree(r->d_enc_sym);
    cudaFree(r->d_enc_slot);
    cudaFree(r->d_cost);
    cudaFree(r->d_amax);
    cudaFree(r->d_runs);
    cudaFree(r->d_desc);
    cudaFree(r->d_slots);
    cudaFree(r->d_stats);
    cudaFree(r->d_list);
    cudaFree(r->d_count);
    cudaFree(r->d_status);
    cudaFreeHost(r->h_len);
    cudaFreeHost(r->h_ptr);
    cudaFreeHost(r->h_status);
    delete r;
}

int check_geometry(int64_t scan_rows, int64_t scan_cols, int32_t det_rows, int32_t det_cols, int32_t bits)
{
    if (scan_rows <= 0 || scan_cols <= 0 || det_rows <= 0 || det_cols <= 0)
        return QEM_ERR_ARG;
    if ((scan_rows * scan_cols) % kScans != 0)
        return QEM_ERR_ARG;
    if (static_cast<int64_t>(det_rows) * det_cols >= (int64_t(1) << 24))
        return QEM_ERR_ARG;
    if (bits != 8 && bits != 16)
        return QEM_ERR_ARG;
    return QEM_OK;
}

int make_resident(int64_t scan_rows, int64_t scan_cols, int32_t det_rows, int32_t det_cols, int32_t bits,
                  const uint8_t *valid, bool valid_on_host, cudaStream_t st, qem_resident **out)
{
    *out = nullptr;
    int rc = check_geometry(scan_rows, scan_cols, det_rows, det_cols, bits);
    if (rc)
        return rc;
    qem_resident *r = new qem_resident();
    auto fail = [&](int code) {
        release(r);
        return code;
    };
    cudaGetDevice(&r->device);
    cudaDeviceGetAttribute(&r->n_sm, cudaDevAttrMultiProcessorCount, r->device);
    r->scan_rows = scan_rows;
    r->scan_cols = scan_cols;
    r->det_rows = det_rows;
    r->det_cols = det_cols;
    r->bits = bits;
    r->w = bits / 8;
    r->P = det_rows * det_cols;
    r->G = (r->P + 31) / 32;
    r->B = scan_rows * scan_cols / kScans;
    r->blk_len.assign(static_cast<size_t>(r->B), 0);
    r->blk_ptr.assign(static_cast<size_t>(r->B), 0);

    std::vector<uint8_t> hv(static_cast<size_t>(r->P), 1);
    if (valid) {
        const cudaError_t e = valid_on_host
                                  ? (std::memcpy(hv.data(), valid, hv.size()), cudaSuccess)
                                  : cudaMemcpy(hv.data(), valid, hv.size(), cudaMemcpyDeviceToHost);
        if (e != cudaSuccess)
            return fail(cuda_status(e));
    }
    r->n_valid = 0;
    for (auto &x : hv) {
        x = x ? 1 : 0;
        r->n_valid += x;
    }
    r->h_valid = hv;
    r->out_bits_auto = static_cast<uint64_t>(r->n_valid) * ((1ull << bits) - 1ull) > 0xFFFFFFFFull ? 64 : 32;

    const HostTables &T = host_tables();
    if ((rc = dalloc(&r->d_valid, hv.size())) || (rc = dalloc(&r->d_pclass, hv.size())) || (rc = dalloc(&r->d_groups, size_t(r->B) * r->G * kGroupWords * 4)) ||
        (rc = dalloc(&r->d_blk_ptr, size_t(r->B) * 8)) || (rc = dalloc(&r->d_blk_len, size_t(r->B) * 4)) ||
        (rc = dalloc(&r->d_dec, sizeof(T.dec))) || (rc = dalloc(&r->d_enc_sym, sizeof(T.enc_sym))) ||
        (rc = dalloc(&r->d_enc_slot, sizeof(T.enc_slot))) || (rc = dalloc(&r->d_cost, sizeof(T.cost))) ||
        (rc = dalloc(&r->d_amax, kModels * 4)) || (rc = dalloc(&r->d_runs, sizeof(T.runs))) || (rc = dalloc(&r->d_stats, (5 + kModels) * 8)) ||
        (rc = dalloc(&r->d_list, size_t(r->P) * 4)) || (rc = dalloc(&r->d_count, 32)) ||
        (rc = dalloc(&r->d_status, sizeof(DevStatus))))
        return fail(rc);
    if (cudaMemset(r->d_count, 0, 32) != cudaSuccess)
        return fail(QEM_ERR_CUDA);
    if (cudaMallocHost(&r->h_status, sizeof(DevStatus)) != cudaSuccess)
        return fail(QEM_ERR_OOM);
    std::memset(r->h_status, 0, sizeof(DevStatus));
    uint32_t amax[kModels];
    for (int m = 0; m < kModels; ++m)
        amax[m] = T.amax[m];
    cudaError_t e = cudaSuccess;
    auto up = [&](void *d, const void *h, size_t n) {
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(d, h, n, cudaMemcpyHostToDevice, st);
    };
    up(r->d_valid, hv.data(), hv.size());
    up(r->d_dec, T.dec, sizeof(T.dec));
    up(r->d_enc_sym, T.enc_sym, sizeof(T.enc_sym));
    up(r->d_enc_slot, T.enc_slot, sizeof(T.enc_slot));
    up(r->d_cost, T.cost, sizeof(T.cost));
    up(r->d_amax, amax, sizeof(amax));
    up(r->d_runs, T.runs, sizeof(T.runs));
    r->skip_models = T.skip_models;
    if (e == cudaSuccess)
        e = cudaMemsetAsync(r->d_pclass, 0, hv.size(), st);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(r->d_stats, 0, (5 + kModels) * 8, st);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(r->d_status, 0, sizeof(DevStatus), st);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(r->d_groups, 0, size_t(r->B) * r->G * kGroupWords * 4, st);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(st);        // host staging above goes out of scope
    if (e != cudaSuccess)
        return fail(cuda_status(e));
    // set-up of the allocation-free masked sum on this device (its working array
    // and kernels are loaded here, when allocating is expected, not at its first call);
    // a failure leaves that one entry point unavailable, not the resident
    if (noalloc_setup(r->device, &r->noalloc_scratch, &r->noalloc_flags) != QEM_OK) {
        r->noalloc_scratch = nullptr;
        r->noalloc_flags = nullptr;
        cudaGetLastError();
    }
    *out = r;
    return QEM_OK;
}

// Place a block of `len` bytes in an arena (new arena when the current is full).
int place_block(qem_resident *r, int64_t b, uint64_t len, unsigned long long &ptr)
{
    const size_t need = static_cast<size_t>(len) + kArenaPad;
    if (r->arenas.empty() || r->arenas.back().used + need > r->arenas.back().cap) {
        const size_t bound_rest = static_cast<size_t>(r->B - b) * r->P * (2 + kScans * r->w) + kArenaPad;
        size_t cap = bound_rest < kArenaMax ? bound_rest : kArenaMax;
        if (cap < need)
            cap = need;
        cap = (cap + 255) & ~size_t(255);
        Arena a;
        void *p = nullptr;
        QEM_CK(cudaMalloc(&p, cap));
        a.p = static_cast<uint8_t *>(p);
        a.cap = cap;
        a.used = 0;
        r->arenas.push_back(a);
        QEM_CK(cudaMemset(a.p, 0, cap));
    }
    Arena &a = r->arenas.back();
    ptr = reinterpret_cast<unsigned long long>(a.p + a.used);
    a.used = (a.used + static_cast<size_t>(len) + 15) & ~size_t(15);
    return QEM_OK;
}

int ensure_scratch(qem_resident *r, int nblk)
{
    const size_t streams = static_cast<size_t>(nblk) * r->P;
    if (streams > r->scratch_streams) {
        cudaFree(r->d_desc);
        cudaFree(r->d_slots);
        r->d_desc = nullptr;
        r->d_slots = nullptr;
        r->scratch_streams = 0;
        int rc;
        if ((rc = dalloc(&r->d_desc, streams * sizeof(uint4))) ||
            (rc = dalloc(&r->d_slots, streams * kSlotWords * sizeof(uint32_t))))
            return rc;
        r->scratch_streams = streams;
    }
    if (static_cast<size_t>(nblk) > r->pinned_blocks) {
        cudaFreeHost(r->h_len);
        cudaFreeHost(r->h_ptr);
        r->h_len = nullptr;
        r->h_ptr = nullptr;
        r->pinned_blocks = 0;
        QEM_CK(cudaMallocHost(&r->h_len, static_cast<size_t>(nblk) * 4));
        QEM_CK(cudaMallocHost(&r->h_ptr, static_cast<size_t>(nblk) * 8));
        r->pinned_blocks = static_cast<size_t>(nblk);
    }
    return QEM_OK;
}

int collect_stats(qem_resident *r, cudaStream_t st)
{
    unsigned long long h[5 + kModels];
    QEM_CK(cudaMemcpyAsync(h, r->d_stats, sizeof(h), cudaMemcpyDeviceToHost, st));
    QEM_CK(cudaStreamSynchronize(st));
    for (int i = 0; i < 5; ++i)
        r->form_count[i] += h[i];
    for (int m = 0; m < kModels; ++m)
        r->model_count[m] += h[5 + m];
    QEM_CK(cudaMemsetAsync(r->d_stats, 0, sizeof(h), st));
    return QEM_OK;
}

int report_errors(qem_resident *r, cudaStream_t st)
{
    if (r->h_status->flags == 0u) {
        for (auto &kv : r->baselines)
            kv.second.pending = false;
        return QEM_OK;
    }
    for (auto &kv : r->baselines)
        if (kv.second.pending) {
            kv.second.state = kTainted;
            kv.second.pending = false;
        }
    const bool timed_out = (r->h_status->flags & kErrWait) != 0u;
    const unsigned long long rows = r->h_status->rows, streams = r->h_status->streams;
    std::memset(r->h_status, 0, sizeof(DevStatus));
    r->h_status->rows = rows;
    r->h_status->streams = streams;
    QEM_CK(cudaMemcpyAsync(r->d_status, r->h_status, sizeof(DevStatus), cudaMemcpyHostToDevice, st));
    QEM_CK(cudaStreamSynchronize(st));
    return timed_out ? QEM_ERR_TIMEOUT : QEM_ERR_MALFORMED;
}

// The cached full-detector image of the complement queries: every valid
// pixel's stream decoded once (plan over the validity map, no baseline
// touched), [B][512] uint64.  Synchronous on first use; a malformed stream
// leaves no cache.
int compute_total(qem_resident *r, cudaStream_t st)
{
    if (r->total_ready)
        return QEM_OK;
    int rc;
    if ((!r->d_total && (rc = dalloc(&r->d_total, static_cast<size_t>(r->B) * kScans * 8))) ||
        (!r->d_tot_mask && (rc = dalloc(&r->d_tot_mask, static_cast<size_t>(r->P)))))
        return rc;
    uint32_t *count = r->d_count + 4 * r->count_pair;
    uint32_t *count_next = r->d_count + 4 * (r->count_pair ^ 1);
    rc = timed(r, QEM_K_PLAN, st, [&] {
        return launch_plan(r->d_valid, r->d_valid, r->d_pclass, r->d_tot_mask, r->P, 0, r->d_list, count, count_next,
                           r->d_total, nullptr, r->B * kScans, 8, st);
    });
    if (rc)
        return rc;
    r->count_pair ^= 1;
    rc = timed(r, QEM_K_DECODE_REDUCE, st, [&] {
        return launch_decode_reduce(r->view(), r->tables(), r->d_list, count, 1, r->B, r->d_total, 8, r->d_status,
                                    r->n_sm, st);
    });
    if (rc)
        return rc;
    QEM_CK(cudaMemcpyAsync(r->h_status, r->d_status, sizeof(DevStatus), cudaMemcpyDeviceToHost, st));
    if ((rc = bounded_wait(st)))
        return rc;
    if (r->h_status->flags)
        return report_errors(r, st);
    r->total_ready = true;
    return QEM_OK;
}

int query(qem_resident *r, const uint8_t *d_mask, int32_t k, int32_t out_bits, void *d_out, int32_t *used,
          int32_t wait, cudaStream_t st, bool delta, bool complement = false)
{
    if (!r || !d_mask || !d_out || k < 1 || (reinterpret_cast<uintptr_t>(d_out) & 15u))
        return QEM_ERR_ARG;
    if (r->B_done != r->B)
        return QEM_ERR_STATE;
    int bits;
    if (out_bits == 0)
        bits = r->out_bits_auto;
    else if (out_bits == 64)
        bits = 64;
    else if (out_bits == 32 && r->out_bits_auto == 32)
        bits = 32;
    else
        return QEM_ERR_ARG;
    const long long rows = (r->B + k - 1) / k;
    const long long n_elems = rows * kScans;

    Baseline &bl = r->baselines[k];
    if (!bl.d_mask) {
        int rc;
        if ((rc = dalloc(&bl.d_mask, r->P)) || (rc = dalloc(&bl.d_img, static_cast<size_t>(n_elems) * 8)))
            return rc;
        QEM_CK(cudaMemsetAsync(bl.d_mask, 0, r->P, st));
    }
    int mode = 0;
    if (delta) {
        if (bl.state == kTainted)
            return QEM_ERR_TAINTED;
        if (bl.state == kValid && bl.out_bits == bits)
            mode = 1;
    }
    if (complement) {
        int rc0 = compute_total(r, st);
        if (rc0)
            return rc0;
        mode = 2;
    }
    uint32_t *count = r->d_count + 4 * r->count_pair;
    uint32_t *count_next = r->d_count + 4 * (r->count_pair ^ 1);
    // The index plan serves full queries; a delta lists its changed pixels one by
    // one (a moving mask changes pixels along its edge, which rarely fill a whole
    // group, and the per-pixel plan is the shorter launch).
    const bool use_index = r->has_index && mode == 0 && !complement;
    int rc = timed(r, QEM_K_PLAN, st, [&] {
        if (use_index)
            return launch_plan_index(d_mask, r->d_pclass, bl.d_mask, r->P, mode, r->d_idx_slots, r->d_idx_root_leaf0,
                                     r->idx_R, r->d_list, r->d_idx_items, count, count_next, d_out, bl.d_img,
                                     n_elems, bits / 8, st);
        return launch_plan(d_mask, r->d_valid, r->d_pclass, bl.d_mask, r->P, mode, r->d_list, count, count_next,
                           d_out, bl.d_img, n_elems, bits / 8, st, r->d_total, k);
    });
    if (rc)
        return rc;
    r->count_pair ^= 1;
    // the decode adds every term to d_out and to the stride's kept image, so
    // the kept image is this query's result without a copy
    rc = timed(r, QEM_K_DECODE_REDUCE, st, [&] {
        const IndexView ix = use_index ? IndexView{r->d_idx_desc, r->d_idx_base, r->d_idx_items, r->idx_L,
                                                      r->idx_L + r->idx_R}
                                          : IndexView{nullptr, nullptr, nullptr, 0, 0};
        // the index plan may list pixels with a minus sign (a leaf's stored sums minus
        // its unmasked pixels), so its queries take the signed decode
        return launch_decode_reduce(r->view(), r->tables(), r->d_list, count, k, rows, d_out, bits / 8,
                                    r->d_status, r->n_sm, st, mode == 1, bl.d_img, ix, mode != 0 || use_index);
    });
    if (rc)
        return rc;
    bl.state = kValid;
    bl.out_bits = bits;
    bl.pending = true;
    if (used)
        *used = bits;
    if (wait) {
        // queued (wait == 0) queries leave the status on the device; it accumulates
        // until qem_finish copies it back
        QEM_CK(cudaMemcpyAsync(r->h_status, r->d_status, sizeof(DevStatus), cudaMemcpyDeviceToHost, st));
        rc = bounded_wait(st);
        if (rc)
            return rc;
        return report_errors(r, st);
    }
    return QEM_OK;
}

// Polar layout of the interaction index (page "Operation pipeline" step 3:
// radial-angular pixel groups, 64-pixel leaves, 16-leaf roots).  Reading:
// the valid pixels are split into 16 angular sectors around the centre
// (boundaries every 22.5 degrees, so the row and column axes through the
// centre are sector edges), ordered by distance inside each sector (then by
// angle and index), and cut into leaves of 64 consecutive pixels; 16
// consecutive leaves of one sector form a root.  A disk or annulus about the
// centre then covers whole leaves and roots except along its two circles, and
// a quadrant of one covers whole leaves except along its arc.
struct PolarLayout {
    std::vector<uint32_t> slots;     // [64 L], padding = P
    std::vector<int> root_leaf0;     // [R + 1]
    int L = 0, R = 0;
};

PolarLayout polar_layout(int det_rows, int det_cols, const std::vector<uint8_t> &valid, double cr, double cc)
{
    constexpr int kSectors = 16;
    const double two_pi = 6.283185307179586;
    struct Px {
        int sector;
        double d2, ang;
        int p;
    };
    std::vector<std::vector<Px>> sec(kSectors);
    for (int r = 0; r < det_rows; ++r)
        for (int c = 0; c < det_cols; ++c) {
            const int p = r * det_cols + c;
            if (!valid[p])
                continue;
            const double dr = r - cr, dc = c - cc;
            double a = std::atan2(dr, dc);          // (-pi, pi]
            if (a < 0)
                a += two_pi;                        // [0, 2 pi)
            int s = static_cast<int>(a / (two_pi / kSectors));
            s = s < 0 ? 0 : (s >= kSectors ? kSectors - 1 : s);
            sec[s].push_back(Px{s, dr * dr + dc * dc, a, p});
        }
    PolarLayout out;
    const uint32_t P = static_cast<uint32_t>(det_rows) * static_cast<uint32_t>(det_cols);
    for (auto &v : sec) {
        std::sort(v.begin(), v.end(), [](const Px &x, const Px &y) {
            if (x.d2 != y.d2)
                return x.d2 < y.d2;
            if (x.ang != y.ang)
                return x.ang < y.ang;
            return x.p < y.p;
        });
        const int leaves = static_cast<int>((v.size() + 63) / 64);
        for (int l = 0; l < leaves; ++l) {
            if (l % 16 == 0)
                out.root_leaf0.push_back(out.L);
            for (int k = 0; k < 64; ++k) {
                const size_t i = static_cast<size_t>(l) * 64 + k;
                out.slots.push_back(i < v.size() ? static_cast<uint32_t>(v[i].p) : P);
            }
            ++out.L;
        }
    }
    out.R = static_cast<int>(out.root_leaf0.size());
    out.root_leaf0.push_back(out.L);
    return out;
}

void drop_index(qem_resident *r)
{
    for (auto &a : r->idx_arenas)
        cudaFree(a.p);
    r->idx_arenas.clear();
    cudaFree(r->d_idx_slots);
    cudaFree(r->d_idx_root_leaf0);
    cudaFree(r->d_idx_desc);
    cudaFree(r->d_idx_base);
    cudaFree(r->d_idx_items);
    r->d_idx_slots = nullptr;
    r->d_idx_root_leaf0 = nullptr;
    r->d_idx_desc = nullptr;
    r->d_idx_base = nullptr;
    r->d_idx_items = nullptr;
    r->has_index = false;
    r->idx_L = r->idx_R = 0;
    r->idx_bytes = 0;
}

// Reserve n bytes (512-aligned) of index storage; returns the device address.
int place_index(qem_resident *r, uint64_t n, unsigned long long &ptr)
{
    const uint64_t need = (n + 511) & ~uint64_t(511);
    if (r->idx_arenas.empty() || r->idx_arenas.back().used + need > r->idx_arenas.back().cap) {
        Arena a;
        a.cap = std::max<size_t>(need, size_t(256) << 20);
        void *q = nullptr;
        if (cudaMalloc(&q, a.cap) != cudaSuccess)
            return QEM_ERR_OOM;
        a.p = static_cast<uint8_t *>(q);
        r->idx_arenas.push_back(a);
    }
    Arena &a = r->idx_arenas.back();
    ptr = reinterpret_cast<unsigned long long>(a.p + a.used);
    a.used += need;
    r->idx_bytes += n;
    return QEM_OK;
}

int build_index(qem_resident *r, double cr, double cc, cudaStream_t st)
{
    drop_index(r);
    PolarLayout lay = polar_layout(r->det_rows, r->det_cols, r->h_valid, cr, cc);
    r->idx_L = lay.L;
    r->idx_R = lay.R;
    r->idx_center[0] = cr;
    r->idx_center[1] = cc;
    const int L = lay.L, R = lay.R, G = L + R;
    if (L == 0)
        return QEM_OK;      // no valid pixels: nothing to index
    int rc;
    if ((rc = dalloc(&r->d_idx_slots, lay.slots.size() * 4)) ||
        (rc = dalloc(&r->d_idx_root_leaf0, lay.root_leaf0.size() * 4)) ||
        (rc = dalloc(&r->d_idx_desc, static_cast<size_t>(r->B) * G * 4)) ||
        (rc = dalloc(&r->d_idx_base, static_cast<size_t>(r->B) * 8)) ||
        (rc = dalloc(&r->d_idx_items, static_cast<size_t>(G) * 4)))
        return rc;
    QEM_CK(cudaMemcpyAsync(r->d_idx_slots, lay.slots.data(), lay.slots.size() * 4, cudaMemcpyHostToDevice, st));
    QEM_CK(cudaMemcpyAsync(r->d_idx_root_leaf0, lay.root_leaf0.data(), lay.root_leaf0.size() * 4,
                           cudaMemcpyHostToDevice, st));
    // blocks per batch: leaf sums of about 64 MB
    const size_t per_block = static_cast<size_t>(L) * kScans * 4;
    int64_t nb = static_cast<int64_t>((size_t(64) << 20) / per_block);
    nb = nb < 1 ? 1 : (nb > r->B ? r->B : nb);
    nb = nb > 32768 ? 32768 : nb;           // grid y of the pack kernel
    uint32_t *leafsum = nullptr;
    unsigned long long *d_total = nullptr;
    std::vector<unsigned long long> total(static_cast<size_t>(nb)), base(static_cast<size_t>(r->B));
    auto cleanup = [&](int code) {
        cudaFree(leafsum);
        cudaFree(d_total);
        if (code != QEM_OK)
            drop_index(r);
        return code;
    };
    if ((rc = dalloc(&leafsum, per_block * nb)) || (rc = dalloc(&d_total, static_cast<size_t>(nb) * 8)))
        return cleanup(rc);
    for (int64_t b0 = 0; b0 < r->B; b0 += nb) {
        const int n = static_cast<int>(std::min<int64_t>(nb, r->B - b0));
        cudaError_t e = cudaMemsetAsync(leafsum, 0, per_block * n, st);
        if (e == cudaSuccess)
            e = launch_index_sums(r->view(), r->tables(), r->d_idx_slots, L, b0, n, leafsum, r->d_status, r->n_sm, st);
        if (e == cudaSuccess)
            e = launch_index_size(leafsum, r->d_idx_root_leaf0, L, G, n, r->d_idx_desc + b0 * G, d_total, st);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(total.data(), d_total, static_cast<size_t>(n) * 8, cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess)
            e = cudaStreamSynchronize(st);
        if (e != cudaSuccess)
            return cleanup(cuda_status(e));
        for (int i = 0; i < n; ++i)
            if ((rc = place_index(r, total[i], base[b0 + i])))
                return cleanup(rc);
        e = cudaMemcpyAsync(r->d_idx_base + b0, base.data() + b0, static_cast<size_t>(n) * 8, cudaMemcpyHostToDevice,
                            st);
        if (e == cudaSuccess)
            e = launch_index_pack(leafsum, r->d_idx_root_leaf0, L, G, b0, n, r->d_idx_desc, r->d_idx_base, st);
        if (e != cudaSuccess)
            return cleanup(cuda_status(e));
    }
    // malformed streams met while summing make the index unusable
    QEM_CK(cudaMemcpyAsync(r->h_status, r->d_status, sizeof(DevStatus), cudaMemcpyDeviceToHost, st));
    if ((rc = bounded_wait(st)))
        return cleanup(rc);
    if (r->h_status->flags) {
        rc = report_errors(r, st);
        return cleanup(rc ? rc : QEM_ERR_MALFORMED);
    }
    r->has_index = true;
    return cleanup(QEM_OK);
}

}  // namespace

namespace qem {
int bounded_stream_wait(cudaStream_t st)
{
    const auto t0 = std::chrono::steady_clock::now();
    for (;;) {
        const cudaError_t e = cudaStreamQuery(st);
        if (e == cudaSuccess)
            return QEM_OK;
        if (e != cudaErrorNotReady)
            return cuda_status(e);
        const double dt = std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
        if (dt > kWaitSeconds)
            return QEM_ERR_TIMEOUT;
        std::this_thread::sleep_for(std::chrono::microseconds(dt < 0.01 ? 2 : 200));
    }
}
}  // namespace qem

extern "C" {

const char *qem_abi(void) { return "qem-pair-v2"; }

const char *qem_status_string(int s)
{
    switch (s) {
    case QEM_OK: return "ok";
    case QEM_ERR_ARG: return "invalid argument";
    case QEM_ERR_MALFORMED: return "malformed stream";
    case QEM_ERR_CUDA: return "CUDA error";
    case QEM_ERR_OOM: return "out of device memory";
    case QEM_ERR_TIMEOUT: return "device wait timed out";
    case QEM_ERR_TAINTED: return "delta baseline invalidated by a failed decode";
    case QEM_ERR_STATE: return "resident not complete";
    default: return "unknown status";
    }
}

int qem_create(int64_t scan_rows, int64_t scan_cols, int32_t det_rows, int32_t det_cols, int32_t dtype_bits,
               const uint8_t *d_valid, void *stream, qem_resident **out)
{
    if (!out)
        return QEM_ERR_ARG;
    return make_resident(scan_rows, scan_cols, det_rows, det_cols, dtype_bits, d_valid, false,
                         static_cast<cudaStream_t>(stream), out);
}

int qem_encode_append(qem_resident *r, const void *d_counts, int64_t n_blocks, void *stream)
{
    if (!r || !d_counts || n_blocks < 0 || r->B_done + n_blocks > r->B ||
        (reinterpret_cast<uintptr_t>(d_counts) & static_cast<uintptr_t>(r->w - 1)))
        return QEM_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t block_raw = static_cast<size_t>(kScans) * r->P * r->w;
    int64_t per = static_cast<int64_t>(kBatchRawBytes / block_raw);
    if (per < 1)
        per = 1;
    if (per > n_blocks)
        per = n_blocks > 0 ? n_blocks : 1;
    int rc = ensure_scratch(r, static_cast<int>(per));
    if (rc)
        return rc;
    const uint8_t *src = static_cast<const uint8_t *>(d_counts);
    for (int64_t done = 0; done < n_blocks;) {
        const int nb = static_cast<int>(n_blocks - done < per ? n_blocks - done : per);
        const void *counts = src + static_cast<size_t>(done) * block_raw;
        const int64_t b0 = r->B_done;
        rc = timed(r, QEM_K_ENC_STREAMS, st, [&] {
            return launch_enc_streams(counts, r->w, r->P, nb, r->tables(), r->d_desc, r->d_slots, r->d_stats,
                                      b0 == 0 ? r->d_pclass : nullptr, st);
        });
        if (rc)
            return rc;
        rc = timed(r, QEM_K_ENC_LAYOUT, st, [&] {
            return launch_enc_layout(r->d_desc, r->P, r->G, nb, r->d_groups + size_t(b0) * r->G * kGroupWords,
                                     r->d_blk_len + b0, st);
        });
        if (rc)
            return rc;
        QEM_CK(cudaMemcpyAsync(r->h_len, r->d_blk_len + b0, size_t(nb) * 4, cudaMemcpyDeviceToHost, st));
        QEM_CK(cudaStreamSynchronize(st));
        for (int i = 0; i < nb; ++i) {
            unsigned long long ptr;
            if ((rc = place_block(r, b0 + i, r->h_len[i], ptr)))
                return rc;
            r->h_ptr[i] = ptr;
            r->blk_len[b0 + i] = r->h_len[i];
            r->blk_ptr[b0 + i] = ptr;
        }
        QEM_CK(cudaMemcpyAsync(r->d_blk_ptr + b0, r->h_ptr, size_t(nb) * 8, cudaMemcpyHostToDevice, st));
        rc = timed(r, QEM_K_ENC_COMPACT, st, [&] {
            return launch_enc_compact(counts, r->w, r->P, nb, r->d_desc, r->d_slots, r->d_blk_ptr + b0, st);
        });
        if (rc)
            return rc;
        r->B_done += nb;
        done += nb;
    }
    return collect_stats(r, st);
}

int qem_encode(const void *d_counts, int32_t dtype_bits, int64_t scan_rows, int64_t scan_cols, int32_t det_rows,
               int32_t det_cols, const uint8_t *d_valid, void *stream, qem_resident **out)
{
    if (!out || !d_counts)
        return QEM_ERR_ARG;
    int rc = qem_create(scan_rows, scan_cols, det_rows, det_cols, dtype_bits, d_valid, stream, out);
    if (rc)
        return rc;
    rc = qem_encode_append(*out, d_counts, (*out)->B, stream);
    if (rc == QEM_OK)
        rc = cuda_status(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    if (rc) {
        release(*out);
        *out = nullptr;
    }
    return rc;
}

int qem_masked_sum(qem_resident *r, const uint8_t *d_mask, int32_t k, int32_t out_bits, void *d_out,
                   int32_t *used, int32_t wait, void *stream)
{
    return query(r, d_mask, k, out_bits, d_out, used, wait, static_cast<cudaStream_t>(stream), false);
}

int qem_masked_sum_delta(qem_resident *r, const uint8_t *d_mask, int32_t k, int32_t out_bits, void *d_out,
                         int32_t *used, int32_t wait, void *stream)
{
    return query(r, d_mask, k, out_bits, d_out, used, wait, static_cast<cudaStream_t>(stream), true);
}

int qem_masked_sum_complement(qem_resident *r, const uint8_t *d_mask, int32_t k, int32_t out_bits, void *d_out,
                              int32_t *used, int32_t wait, void *stream)
{
    return query(r, d_mask, k, out_bits, d_out, used, wait, static_cast<cudaStream_t>(stream), false, true);
}

int qem_decode_blocks(qem_resident *r, int64_t first, int64_t n, void *d_out, int32_t wait, void *stream)
{
    if (!r || !d_out || first < 0 || n < 0 || first + n > r->B_done ||
        (reinterpret_cast<uintptr_t>(d_out) & static_cast<uintptr_t>(r->w - 1)))
        return QEM_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (n == 0)
        return QEM_OK;
    int rc = timed(r, QEM_K_DECODE_BLOCKS, st, [&] {
        return launch_decode_blocks(r->view(), r->tables(), first, n, d_out, r->d_status, st);
    });
    if (rc)
        return rc;
    if (wait) {
        QEM_CK(cudaMemcpyAsync(r->h_status, r->d_status, sizeof(DevStatus), cudaMemcpyDeviceToHost, st));
        rc = bounded_wait(st);
        if (rc)
            return rc;
        return report_errors(r, st);
    }
    return QEM_OK;
}

int qem_decode_range(qem_resident *r, int64_t first_scan, int64_t n_scans, void *d_out, int32_t wait, void *stream)
{
    if (!r || first_scan < 0 || n_scans < 0 || first_scan + n_scans > r->B_done * kScans)
        return QEM_ERR_ARG;
    if (n_scans == 0)
        return QEM_OK;
    if (!d_out || (reinterpret_cast<uintptr_t>(d_out) & static_cast<uintptr_t>(r->w - 1)))
        return QEM_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc = timed(r, QEM_K_DECODE_BLOCKS, st, [&] {
        return launch_decode_range(r->view(), r->tables(), first_scan, n_scans, d_out, r->d_status, st);
    });
    if (rc)
        return rc;
    if (wait) {
        QEM_CK(cudaMemcpyAsync(r->h_status, r->d_status, sizeof(DevStatus), cudaMemcpyDeviceToHost, st));
        rc = bounded_wait(st);
        if (rc)
            return rc;
        return report_errors(r, st);
    }
    return QEM_OK;
}

int qem_masked_moments(qem_resident *r, const uint8_t *d_mask, const int32_t *d_weights, int32_t k, int64_t *d_out,
                       int32_t wait, void *stream)
{
    if (!r || !d_mask || !d_weights || !d_out || k < 1 || (reinterpret_cast<uintptr_t>(d_out) & 7u) ||
        (reinterpret_cast<uintptr_t>(d_weights) & 3u))
        return QEM_ERR_ARG;
    if (r->B_done != r->B)
        return QEM_ERR_STATE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc;
    if (!r->d_mom_mask && (rc = dalloc(&r->d_mom_mask, static_cast<size_t>(r->P))))
        return rc;
    const long long rows = (r->B + k - 1) / k;
    uint32_t *count = r->d_count + 4 * r->count_pair;
    uint32_t *count_next = r->d_count + 4 * (r->count_pair ^ 1);
    rc = timed(r, QEM_K_PLAN, st, [&] {
        return launch_plan(d_mask, r->d_valid, r->d_pclass, r->d_mom_mask, r->P, 0, r->d_list, count, count_next,
                           nullptr, nullptr, 0, 8, st);
    });
    if (rc)
        return rc;
    r->count_pair ^= 1;
    rc = timed(r, QEM_K_DECODE_REDUCE, st, [&] {
        return launch_moments(r->view(), r->tables(), r->d_list, count, d_weights, k, rows,
                              reinterpret_cast<long long *>(d_out), r->d_status, st);
    });
    if (rc)
        return rc;
    if (wait) {
        QEM_CK(cudaMemcpyAsync(r->h_status, r->d_status, sizeof(DevStatus), cudaMemcpyDeviceToHost, st));
        rc = bounded_wait(st);
        if (rc)
            return rc;
        return report_errors(r, st);
    }
    return QEM_OK;
}

int qem_decode_blocks_amplitude(qem_resident *r, int64_t first, int64_t n, void *d_counts, float *d_amp,
                                int32_t wait, void *stream)
{
    if (!r || !d_amp || (reinterpret_cast<uintptr_t>(d_amp) & 3u))
        return QEM_ERR_ARG;
    int rc = qem_decode_blocks(r, first, n, d_counts, 0, stream);
    if (rc)
        return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (n > 0)
        QEM_CK(launch_amplitude(d_counts, r->w, d_amp, static_cast<long long>(n) * kScans * r->P, st));
    if (wait) {
        QEM_CK(cudaMemcpyAsync(r->h_status, r->d_status, sizeof(DevStatus), cudaMemcpyDeviceToHost, st));
        rc = bounded_wait(st);
        if (rc)
            return rc;
        return report_errors(r, st);
    }
    return QEM_OK;
}

int qem_finish(qem_resident *r, void *stream)
{
    if (!r)
        return QEM_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    QEM_CK(cudaMemcpyAsync(r->h_status, r->d_status, sizeof(DevStatus), cudaMemcpyDeviceToHost, st));
    const int rc = bounded_wait(st);
    if (rc)
        return rc;
    return report_errors(r, st);
}

int qem_info(const qem_resident *r, qem_info_t *o)
{
    if (!r || !o)
        return QEM_ERR_ARG;
    std::memset(o, 0, sizeof(*o));
    o->scan_rows = r->scan_rows;
    o->scan_cols = r->scan_cols;
    o->det_rows = r->det_rows;
    o->det_cols = r->det_cols;
    o->dtype_bits = r->bits;
    o->n_pixels = r->P;
    o->n_valid = r->n_valid;
    o->out_bits_auto = r->out_bits_auto;
    o->n_blocks = r->B;
    o->n_blocks_encoded = r->B_done;
    for (int64_t b = 0; b < r->B_done; ++b)
        o->payload_bytes += r->blk_len[b];
    o->group_bytes = static_cast<uint64_t>(r->B) * r->G * kGroupWords * 4;
    uint64_t dev = o->group_bytes + r->B * 12 + r->P + r->P * 4;
    for (auto &a : r->arenas)
        dev += a.cap;
    dev += r->scratch_streams * (sizeof(uint4) + kSlotWords * 4);
    for (auto &kv : r->baselines)
        dev += r->P + static_cast<uint64_t>((r->B + kv.first - 1) / kv.first) * kScans * 8;
    dev += sizeof(HostTables);
    if (r->d_total)
        dev += static_cast<uint64_t>(r->B) * kScans * 8 + r->P;
    if (r->has_index)
        dev += r->idx_bytes + static_cast<uint64_t>(r->B) * (r->idx_L + r->idx_R) * 4 + r->B * 8 +
               static_cast<uint64_t>(r->idx_L) * 64 * 4 + (r->idx_R + 1) * 4 + (r->idx_L + r->idx_R) * 4;
    o->device_bytes = dev;
    for (int i = 0; i < 5; ++i)
        o->form_count[i] = r->form_count[i];
    for (int m = 0; m < kModels; ++m)
        o->model_count[m] = r->model_count[m];
    o->n_arenas = static_cast<int32_t>(r->arenas.size());
    o->index_bytes = r->has_index ? r->idx_bytes : 0;
    o->index_leaves = r->has_index ? r->idx_L : 0;
    o->index_roots = r->has_index ? r->idx_R : 0;
    return QEM_OK;
}

int qem_query_counters(qem_resident *r, uint64_t *rows, uint64_t *streams, void *stream)
{
    if (!r)
        return QEM_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    DevStatus h;
    QEM_CK(cudaMemcpyAsync(&h, r->d_status, sizeof(h), cudaMemcpyDeviceToHost, st));
    QEM_CK(cudaStreamSynchronize(st));
    if (rows)
        *rows = h.rows;
    if (streams)
        *streams = h.streams;
    QEM_CK(cudaMemsetAsync(reinterpret_cast<uint8_t *>(r->d_status) + offsetof(DevStatus, rows), 0,
                           2 * sizeof(unsigned long long), st));
    QEM_CK(cudaStreamSynchronize(st));
    return QEM_OK;
}

int qem_profile(qem_resident *r, int32_t enable)
{
    if (!r)
        return QEM_ERR_ARG;
    r->prof = enable != 0;
    if (enable)
        std::memset(&r->prof_acc, 0, sizeof(r->prof_acc));
    return QEM_OK;
}

int qem_profile_read(qem_resident *r, qem_profile_t *out)
{
    if (!r || !out)
        return QEM_ERR_ARG;
    for (auto &ev : r->events) {
        QEM_CK(cudaEventSynchronize(ev.b));
        float ms = 0.f;
        QEM_CK(cudaEventElapsedTime(&ms, ev.a, ev.b));
        r->prof_acc.ms[ev.kernel] += ms;
        r->prof_acc.launches[ev.kernel] += 1;
        cudaEventDestroy(ev.a);
        cudaEventDestroy(ev.b);
    }
    r->events.clear();
    *out = r->prof_acc;
    return QEM_OK;
}

void qem_free(qem_resident *r)
{
    if (!r)
        return;
    cudaDeviceSynchronize();
    release(r);
}

int qem_block_bytes(const qem_resident *r, int64_t b, uint64_t *nbytes)
{
    if (!r || !nbytes || b < 0 || b >= r->B_done)
        return QEM_ERR_ARG;
    *nbytes = r->blk_len[b];
    return QEM_OK;
}

int qem_export_block(const qem_resident *r, int64_t b, uint32_t *h_groups, uint8_t *h_payload, void *stream)
{
    if (!r || b < 0 || b >= r->B_done)
        return QEM_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (h_groups)
        QEM_CK(cudaMemcpyAsync(h_groups, r->d_groups + size_t(b) * r->G * kGroupWords,
                               size_t(r->G) * kGroupWords * 4, cudaMemcpyDeviceToHost, st));
    if (h_payload && r->blk_len[b])
        QEM_CK(cudaMemcpyAsync(h_payload, reinterpret_cast<const void *>(r->blk_ptr[b]), r->blk_len[b],
                               cudaMemcpyDeviceToHost, st));
    QEM_CK(cudaStreamSynchronize(st));
    return QEM_OK;
}

int qem_import(int64_t scan_rows, int64_t scan_cols, int32_t det_rows, int32_t det_cols, int32_t dtype_bits,
               const uint32_t *h_groups, const uint8_t *h_payload, const uint64_t *h_block_off,
               const uint8_t *h_valid, void *stream, qem_resident **out)
{
    if (!out || !h_groups || !h_payload || !h_block_off)
        return QEM_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    qem_resident *r = nullptr;
    int rc = make_resident(scan_rows, scan_cols, det_rows, det_cols, dtype_bits, h_valid, true, st, &r);
    if (rc)
        return rc;
    auto fail = [&](int code) {
        release(r);
        *out = nullptr;
        return code;
    };
    const uint64_t total = h_block_off[r->B] - h_block_off[0];
    Arena a;
    a.cap = (static_cast<size_t>(total) + kArenaPad + 255) & ~size_t(255);
    void *p = nullptr;
    if (cudaMalloc(&p, a.cap) != cudaSuccess)
        return fail(QEM_ERR_OOM);
    a.p = static_cast<uint8_t *>(p);
    a.used = total;
    r->arenas.push_back(a);
    cudaError_t e = cudaMemset(a.p, 0, a.cap);
    if (e == cudaSuccess && total)
        e = cudaMemcpy(a.p, h_payload + h_block_off[0], total, cudaMemcpyHostToDevice);
    std::vector<uint32_t> lens(static_cast<size_t>(r->B));
    std::vector<uint8_t> pclass0(static_cast<size_t>(r->P), 1);   // empty streams are light
    for (int64_t b = 0; b < r->B; ++b) {
        r->blk_ptr[b] = reinterpret_cast<unsigned long long>(a.p + (h_block_off[b] - h_block_off[0]));
        r->blk_len[b] = h_block_off[b + 1] - h_block_off[b];
        lens[b] = static_cast<uint32_t>(r->blk_len[b]);
        // statistics from the headers, as the encoder would have counted them
        const uint32_t *g = h_groups + size_t(b) * r->G * kGroupWords;
        const uint8_t *pl = h_payload + h_block_off[b];
        for (int px = 0; px < r->P; ++px) {
            const uint32_t *rec = g + size_t(px >> 5) * kGroupWords;
            const int j = px & 31;
            const uint32_t e1 = (rec[1 + j / 2] >> (16 * (j & 1))) & 0xFFFFu;
            const uint32_t e0 = j ? (rec[1 + (j - 1) / 2] >> (16 * ((j - 1) & 1))) & 0xFFFFu : 0u;
            const uint64_t st0 = uint64_t(rec[0]) + e0;
            if (e1 <= e0 || st0 + 2 > r->blk_len[b]) {
                r->form_count[0] += e1 == e0;
                continue;
            }
            const int form = pl[st0] & 7;
            if (b == 0) {
                const uint32_t hdr = pl[st0] | (uint32_t(pl[st0 + 1]) << 8);
                const bool runs = form == kPaired && ((hdr >> 8) & 0x1Fu) == 0u &&
                                  ((r->skip_models >> ((hdr >> 3) & 31u)) & 1u);
                pclass0[px] = (form == kSparse || runs) ? 1 : 0;
            }
            if (form >= 1 && form <= 4) {
                r->form_count[form] += 1;
                if (form == kPaired)
                    r->model_count[(pl[st0] >> 3) & 31] += 1;
            }
        }
    }
    if (e == cudaSuccess)
        e = cudaMemcpy(r->d_groups, h_groups, size_t(r->B) * r->G * kGroupWords * 4, cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
        e = cudaMemcpy(r->d_blk_ptr, r->blk_ptr.data(), size_t(r->B) * 8, cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
        e = cudaMemcpy(r->d_blk_len, lens.data(), size_t(r->B) * 4, cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
        e = cudaMemcpy(r->d_pclass, pclass0.data(), pclass0.size(), cudaMemcpyHostToDevice);
    if (e != cudaSuccess)
        return fail(cuda_status(e));
    r->B_done = r->B;
    *out = r;
    return QEM_OK;
}

int qem_build_index(qem_resident *r, double center_row, double center_col, void *stream)
{
    if (!r || !std::isfinite(center_row) || !std::isfinite(center_col))
        return QEM_ERR_ARG;
    if (r->B_done != r->B)
        return QEM_ERR_STATE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // queries in flight on this stream read the old index
    QEM_CK(cudaStreamSynchronize(st));
    return build_index(r, center_row, center_col, st);
}

int qem_drop_index(qem_resident *r, void *stream)
{
    if (!r)
        return QEM_ERR_ARG;
    QEM_CK(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    drop_index(r);
    return QEM_OK;
}

int qem_polar_layout(int32_t det_rows, int32_t det_cols, const uint8_t *h_valid, double center_row,
                     double center_col, uint32_t *h_slots, int32_t *h_root_leaf0, int32_t *n_leaves,
                     int32_t *n_roots)
{
    if (det_rows <= 0 || det_cols <= 0 || !std::isfinite(center_row) || !std::isfinite(center_col) ||
        static_cast<int64_t>(det_rows) * det_cols > (int64_t(1) << 24) - 1)
        return QEM_ERR_ARG;
    std::vector<uint8_t> valid(static_cast<size_t>(det_rows) * det_cols, 1);
    if (h_valid)
        for (size_t i = 0; i < valid.size(); ++i)
            valid[i] = h_valid[i] ? 1 : 0;
    const PolarLayout lay = polar_layout(det_rows, det_cols, valid, center_row, center_col);
    if (n_leaves)
        *n_leaves = lay.L;
    if (n_roots)
        *n_roots = lay.R;
    if (h_slots)
        std::memcpy(h_slots, lay.slots.data(), lay.slots.size() * 4);
    if (h_root_leaf0)
        std::memcpy(h_root_leaf0, lay.root_leaf0.data(), lay.root_leaf0.size() * 4);
    return QEM_OK;
}

int qem_index_layout(const qem_resident *r, uint32_t *h_slots, int32_t *h_root_leaf0, int32_t *n_leaves,
                     int32_t *n_roots)
{
    if (!r)
        return QEM_ERR_ARG;
    if (!r->has_index)
        return QEM_ERR_STATE;
    if (n_leaves)
        *n_leaves = r->idx_L;
    if (n_roots)
        *n_roots = r->idx_R;
    if (h_slots)
        QEM_CK(cudaMemcpy(h_slots, r->d_idx_slots, static_cast<size_t>(r->idx_L) * 64 * 4, cudaMemcpyDeviceToHost));
    if (h_root_leaf0)
        QEM_CK(cudaMemcpy(h_root_leaf0, r->d_idx_root_leaf0, static_cast<size_t>(r->idx_R + 1) * 4,
                          cudaMemcpyDeviceToHost));
    return QEM_OK;
}

int qem_export_valid(const qem_resident *r, uint8_t *h_valid)
{
    if (!r || !h_valid)
        return QEM_ERR_ARG;
    std::memcpy(h_valid, r->h_valid.data(), r->h_valid.size());
    return QEM_OK;
}

int qem_index_desc(const qem_resident *r, uint32_t *h_desc)
{
    if (!r || !h_desc)
        return QEM_ERR_ARG;
    if (!r->has_index)
        return QEM_ERR_STATE;
    QEM_CK(cudaMemcpy(h_desc, r->d_idx_desc, static_cast<size_t>(r->B) * (r->idx_L + r->idx_R) * 4,
                      cudaMemcpyDeviceToHost));
    return QEM_OK;
}

int qem_pixel_classes(const qem_resident *r, uint8_t *h_class)
{
    if (!r || !h_class)
        return QEM_ERR_ARG;
    QEM_CK(cudaMemcpy(h_class, r->d_pclass, static_cast<size_t>(r->P), cudaMemcpyDeviceToHost));
    return QEM_OK;
}

int qem_model_tables(uint16_t *h_freq, uint8_t *h_amax, uint32_t *h_cost)
{
    const HostTables &T = host_tables();
    if (h_freq)
        std::memcpy(h_freq, T.freq, sizeof(T.freq));
    if (h_amax)
        std::memcpy(h_amax, T.amax, sizeof(T.amax));
    if (h_cost)
        std::memcpy(h_cost, T.cost, sizeof(T.cost));
    return QEM_OK;
}

int qem_generate_counts(void *d_out, int32_t dtype_bits, uint64_t seed, int64_t scan0, int64_t n_scans,
                        int32_t n_pixels, const uint32_t *d_pixel_class, const uint32_t *d_class_desc,
                        const uint64_t *d_thresholds, void *stream)
{
    if (!d_out || !d_pixel_class || !d_class_desc || !d_thresholds || n_scans < 0 || n_pixels <= 0 ||
        (dtype_bits != 8 && dtype_bits != 16))
        return QEM_ERR_ARG;
    return cuda_status(launch_generate(d_out, dtype_bits, seed, scan0, n_scans, n_pixels, d_pixel_class,
                                       d_class_desc, d_thresholds, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// Read-only view of a resident for the allocation-free masked sum (noalloc.cu).
namespace qem {
int resident_query_view(const qem_resident *r, ResidentQuery *q)
{
    if (!r || !q)
        return QEM_ERR_ARG;
    q->view = r->view();
    q->tables = r->tables();
    q->P = r->P;
    q->B = r->B;
    q->complete = r->B_done == r->B;
    q->out_bits_auto = r->out_bits_auto;
    q->n_sm = r->n_sm;
    q->device = r->device;
    q->valid = r->d_valid;
    q->pclass = r->d_pclass;
    q->noalloc_scratch = r->noalloc_scratch;
    q->noalloc_flags = r->noalloc_flags;
    return QEM_OK;
}
}  // namespace qem
