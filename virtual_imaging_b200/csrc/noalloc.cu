// noalloc.cu -- a masked sum that allocates no device memory.
//
// For callers that must not allocate while they query (see
// qem_masked_sum_noalloc in include/qem.h).  Its working memory lives in one
// fixed array among the library's device globals, so the call itself never
// reaches cudaMalloc/cudaFree.  Everything that could allocate -- looking up
// that array's address (which loads this file's module), loading the
// kernels, the pinned word the status comes back through -- happens once per
// device when a resident is created (noalloc_setup), where allocating is
// expected anyway.  The decode itself is the library's fused decode + masked
// reduce (kernels.cu), unchanged.
#include <mutex>

#include "qem_internal.h"

namespace qem {
namespace {

constexpr int kMaxPixels = QEM_NOALLOC_MAX_PIXELS;
constexpr int kMaxDevices = 64;
constexpr int kPlanThreads = 1024;

// Layout of the fixed working memory: error status, list lengths (count =
// heavy entries from the front of the list, reserved[0] = light entries from
// the back), listed pixels.
struct Scratch {
    DevStatus status;
    uint32_t count;
    uint32_t reserved[7];
    uint32_t list[kMaxPixels];
};

// The working memory itself: shared by every call on this device.  In host
// code this name is only a stand-in; kernels get the address that
// cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_scratch[sizeof(Scratch)];

std::mutex g_mu;
uint32_t *g_flags[kMaxDevices] = {};     // pinned status word per device

// CTA 0 clears the status and builds the pixel list of mask && valid: pixels
// whose streams decode pair by pair (pclass 0) ascending from the front,
// lighter ones (empty, sparse, run-decoded) from the back, as the allocating
// plan orders them, so that warps meet one kind of work.  The other CTAs
// clear the output image.
__global__ void __launch_bounds__(kPlanThreads) k_noalloc_plan(const uint8_t *__restrict__ mask,
                                                              const uint8_t *__restrict__ valid,
                                                              const uint8_t *__restrict__ pclass, int P,
                                                              Scratch *__restrict__ s, uint4 *__restrict__ out,
                                                              long long n_vec)
{
    if (blockIdx.x == 0) {
        __shared__ uint32_t s_h[32], s_l[32];
        __shared__ uint32_t s_th, s_tl;
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        if (threadIdx.x == 0) {
            s->status.flags = 0u;
            s->status.rows = 0ull;
            s->status.streams = 0ull;
        }
        // chunks of 1024 consecutive pixels; ballots keep each class in pixel order
        uint32_t nh = 0, nl = 0;
        for (int c0 = 0; c0 < P; c0 += kPlanThreads) {
            const int p = c0 + static_cast<int>(threadIdx.x);
            const bool sel = p < P && mask[p] != 0 && valid[p] != 0;
            const bool light = sel && pclass[p] != 0;
            const unsigned bh = __ballot_sync(0xFFFFFFFFu, sel && !light);
            const unsigned bl = __ballot_sync(0xFFFFFFFFu, light);
            if (lane == 0) {
                s_h[warp] = __popc(bh);
                s_l[warp] = __popc(bl);
            }
            __syncthreads();
            if (warp == 0) {
                const uint32_t vh = s_h[lane], vl = s_l[lane];
                uint32_t ih = vh, il = vl;
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t yh = __shfl_up_sync(0xFFFFFFFFu, ih, o);
                    const uint32_t yl = __shfl_up_sync(0xFFFFFFFFu, il, o);
                    if (lane >= o) {
                        ih += yh;
                        il += yl;
                    }
                }
                s_h[lane] = ih - vh;
                s_l[lane] = il - vl;
                if (lane == 31) {
                    s_th = ih;
                    s_tl = il;
                }
            }
            __syncthreads();
            const unsigned below = (1u << lane) - 1u;
            if (sel && !light)
                s->list[nh + s_h[warp] + __popc(bh & below)] = static_cast<uint32_t>(p);
            if (light)
                s->list[P - 1 - (nl + s_l[warp] + __popc(bl & below))] = static_cast<uint32_t>(p);
            nh += s_th;
            nl += s_tl;
            __syncthreads();
        }
        if (threadIdx.x == 0) {
            s->count = nh;
            s->reserved[0] = nl;
        }
        return;
    }
    const long long stride = static_cast<long long>(gridDim.x - 1) * blockDim.x;
    for (long long i = static_cast<long long>(blockIdx.x - 1) * blockDim.x + threadIdx.x; i < n_vec; i += stride)
        out[i] = make_uint4(0u, 0u, 0u, 0u);
}

}  // namespace

int noalloc_setup(int device, void **scratch, uint32_t **h_flags)
{
    if (device < 0 || device >= kMaxDevices)
        return QEM_ERR_ARG;
    std::lock_guard<std::mutex> lock(g_mu);
    // the array's address on this device (loading this file's module if needed)
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p)
        return QEM_ERR_CUDA;
    // the kernels the call launches, loaded now rather than at its first launch
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, reinterpret_cast<const void *>(k_noalloc_plan));
    if (e == cudaSuccess)
        e = preload_query_kernels();
    if (e != cudaSuccess)
        return QEM_ERR_CUDA;
    // one pinned word per device for the status read-back; taken again if a
    // device reset released the old one
    cudaPointerAttributes pa;
    if (!g_flags[device] || cudaPointerGetAttributes(&pa, g_flags[device]) != cudaSuccess ||
        pa.type != cudaMemoryTypeHost) {
        cudaGetLastError();
        void *h = nullptr;
        if (cudaMallocHost(&h, 64) != cudaSuccess)
            return QEM_ERR_OOM;
        g_flags[device] = static_cast<uint32_t *>(h);
    }
    *scratch = p;
    *h_flags = g_flags[device];
    return QEM_OK;
}

}  // namespace qem

extern "C" int qem_masked_sum_noalloc(qem_resident *res, const uint8_t *d_mask, int32_t block_stride,
                                      int32_t out_bits, void *d_out, void *stream)
{
    using namespace qem;
    ResidentQuery q;
    if (!res || !d_mask || !d_out || block_stride < 1 || (reinterpret_cast<uintptr_t>(d_out) & 15u))
        return QEM_ERR_ARG;
    int rc = resident_query_view(res, &q);
    if (rc)
        return rc;
    if (q.P > kMaxPixels)
        return QEM_ERR_ARG;
    if (!q.complete)
        return QEM_ERR_STATE;
    if (!q.noalloc_scratch || !q.noalloc_flags)
        return QEM_ERR_CUDA;         // its set-up failed when the resident was created
    int bits;
    if (out_bits == 0)
        bits = q.out_bits_auto;
    else if (out_bits == 64)
        bits = 64;
    else if (out_bits == 32 && q.out_bits_auto == 32)
        bits = 32;
    else
        return QEM_ERR_ARG;
    int device = -1;
    if (cudaGetDevice(&device) != cudaSuccess)
        return QEM_ERR_CUDA;
    if (device != q.device)
        return QEM_ERR_ARG;
    Scratch *s = static_cast<Scratch *>(q.noalloc_scratch);

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const long long rows = (q.B + block_stride - 1) / block_stride;
    const long long n_vec = rows * kScans * (bits / 8) / 16;
    int fill = static_cast<int>((n_vec + kPlanThreads - 1) / kPlanThreads);
    fill = fill < 1 ? 1 : (fill > 4 * q.n_sm ? 4 * q.n_sm : fill);
    k_noalloc_plan<<<1 + fill, kPlanThreads, 0, st>>>(d_mask, q.valid, q.pclass, q.P, s,
                                                      static_cast<uint4 *>(d_out), n_vec);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return QEM_ERR_CUDA;
    e = launch_decode_reduce(q.view, q.tables, s->list, &s->count, block_stride, rows, d_out, bits / 8, &s->status,
                             q.n_sm, st);
    if (e != cudaSuccess)
        return QEM_ERR_CUDA;
    *q.noalloc_flags = 0u;
    e = cudaMemcpyAsync(q.noalloc_flags, &s->status.flags, sizeof(uint32_t), cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess)
        return QEM_ERR_CUDA;
    if ((rc = bounded_stream_wait(st)))
        return rc;
    const uint32_t flags = *reinterpret_cast<volatile uint32_t *>(q.noalloc_flags);
    if (flags & kErrWait)
        return QEM_ERR_TIMEOUT;
    return flags ? QEM_ERR_MALFORMED : QEM_OK;
}
