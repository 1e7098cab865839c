// noalloc.cu -- a masked sum that allocates no device memory.
//
// For callers that must not allocate while they query (see
// qem_masked_sum_noalloc in include/qem.h).  Its working memory lives in one
// fixed array among the library's device globals, so the call itself never
// reaches cudaMalloc/cudaFree.  The decode itself is the library's fused
// decode + masked reduce (kernels.cu), unchanged.
#include <mutex>

#include "qem_internal.h"

namespace qem {
namespace {

constexpr int kMaxPixels = QEM_NOALLOC_MAX_PIXELS;
constexpr int kMaxDevices = 64;
constexpr int kPlanThreads = 1024;

// Layout of the fixed working memory: error status, list length (count, then
// reserved[0] = 0 as the decoder's second list segment), listed pixels.
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
void *g_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up once per device).
int scratch_address(int device, Scratch **out)
{
    if (device < 0 || device >= kMaxDevices)
        return QEM_ERR_ARG;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[device]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess || !p)
            return QEM_ERR_CUDA;
        g_addr[device] = p;
    }
    *out = static_cast<Scratch *>(g_addr[device]);
    return QEM_OK;
}

// CTA 0 clears the status and builds the ascending list of pixels with
// mask && valid; the other CTAs clear the output image.
__global__ void __launch_bounds__(kPlanThreads) k_noalloc_plan(const uint8_t *__restrict__ mask,
                                                              const uint8_t *__restrict__ valid, int P,
                                                              Scratch *__restrict__ s, uint4 *__restrict__ out,
                                                              long long n_vec)
{
    if (blockIdx.x == 0) {
        __shared__ uint32_t s_warp[32];
        __shared__ uint32_t s_total;
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        if (threadIdx.x == 0) {
            s->status.flags = 0u;
            s->status.rows = 0ull;
            s->status.streams = 0ull;
        }
        // chunks of 1024 consecutive pixels; ballots keep the list ascending
        uint32_t base = 0;
        for (int c0 = 0; c0 < P; c0 += kPlanThreads) {
            const int p = c0 + static_cast<int>(threadIdx.x);
            const bool sel = p < P && mask[p] != 0 && valid[p] != 0;
            const unsigned bal = __ballot_sync(0xFFFFFFFFu, sel);
            if (lane == 0)
                s_warp[warp] = __popc(bal);
            __syncthreads();
            if (warp == 0) {
                uint32_t v = s_warp[lane];
                uint32_t inc = v;
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, inc, o);
                    if (lane >= o)
                        inc += y;
                }
                s_warp[lane] = inc - v;
                if (lane == 31)
                    s_total = inc;
            }
            __syncthreads();
            if (sel)
                s->list[base + s_warp[warp] + __popc(bal & ((1u << lane) - 1u))] = static_cast<uint32_t>(p);
            base += s_total;
            __syncthreads();
        }
        if (threadIdx.x == 0) {
            s->count = base;
            s->reserved[0] = 0u;     // no light-class entries: the whole list is one segment
        }
        return;
    }
    const long long stride = static_cast<long long>(gridDim.x - 1) * blockDim.x;
    for (long long i = static_cast<long long>(blockIdx.x - 1) * blockDim.x + threadIdx.x; i < n_vec; i += stride)
        out[i] = make_uint4(0u, 0u, 0u, 0u);
}

}  // namespace
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
    Scratch *s = nullptr;
    if ((rc = scratch_address(device, &s)))
        return rc;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const long long rows = (q.B + block_stride - 1) / block_stride;
    const long long n_vec = rows * kScans * (bits / 8) / 16;
    int fill = static_cast<int>((n_vec + kPlanThreads - 1) / kPlanThreads);
    fill = fill < 1 ? 1 : (fill > 4 * q.n_sm ? 4 * q.n_sm : fill);
    k_noalloc_plan<<<1 + fill, kPlanThreads, 0, st>>>(d_mask, q.valid, q.P, s, static_cast<uint4 *>(d_out), n_vec);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e == cudaErrorMemoryAllocation ? QEM_ERR_OOM : QEM_ERR_CUDA;
    e = launch_decode_reduce(q.view, q.tables, s->list, &s->count, block_stride, rows, d_out, bits / 8, &s->status,
                             q.n_sm, st);
    if (e != cudaSuccess)
        return QEM_ERR_CUDA;
    uint32_t flags = 0;
    e = cudaMemcpyAsync(&flags, &s->status.flags, sizeof(flags), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(st);
    if (e != cudaSuccess)
        return QEM_ERR_CUDA;
    if (flags & kErrWait)
        return QEM_ERR_TIMEOUT;
    return flags ? QEM_ERR_MALFORMED : QEM_OK;
}
