// noalloc.cu -- rq_decode_attn_noalloc: decode attention whose split-combine
// scratch lives in a fixed, library-owned device array instead of memory the
// caller or the library has to allocate.
//
// Who needs it: code that must not allocate device memory after start-up --
// a plugin inside a host framework that owns every device byte and offers no
// allocator, a real-time serving loop whose memory is planned once, or work
// issued while a stream is being captured, where an allocation call is
// refused or breaks the capture.  Such a caller still passes its own inputs
// and outputs (the cache, q, out); only the split partials move here.
//
// The array below is a file-scope __device__ object: every GPU that loads this
// library holds kScratchFloats floats (8 MiB) of it until the process exits.
// Host code cannot use its name as a device address, so the first call on each
// device resolves the address with cudaGetSymbolAddress (with that device
// current) and caches it; make that first call before any stream capture.
// All calls on a device share the one array and it keeps the last call's
// contents: calls whose GPU work overlaps (other streams, other threads) race
// on it and must be ordered by the caller.  The split partials need no
// clearing (each slot is written before it is read within a call); the last
// 64 Ki words hold the split-combine counters, zeroed once at set-up and
// returned to zero by every call.
#include <mutex>

#include "rq_internal.h"

namespace {

constexpr size_t kScratchFloats = size_t(2) << 20;   // 2 Mi floats = 8 MiB in all
constexpr size_t kCounterInts = 65536;               // combine counters, at the end of the array
constexpr size_t kPartialFloats = kScratchFloats - kCounterInts;

static __device__ __align__(256) float g_decode_scratch[kScratchFloats];

std::mutex g_setup_mutex;
float *g_scratch_ptr[rq::kMaxDevices] = {nullptr};

// Device address of g_decode_scratch on the current device (resolved once).
int scratch_for_current_device(float **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return RQ_ERR_CUDA;
    if (dev < 0 || dev >= rq::kMaxDevices) return RQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return RQ_ERR_CUDA;
        }
        // the combine counters must start at zero (each call leaves them at zero)
        if (cudaMemset(static_cast<float *>(p) + kPartialFloats, 0, kCounterInts * sizeof(int)) != cudaSuccess ||
            cudaDeviceSynchronize() != cudaSuccess) {
            cudaGetLastError();
            return RQ_ERR_CUDA;
        }
        g_scratch_ptr[dev] = static_cast<float *>(p);
    }
    *out = g_scratch_ptr[dev];
    return RQ_OK;
}

}  // namespace

namespace rq {
void noalloc_reset_counters() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return;
    }
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_ptr[dev]) cudaMemset(g_scratch_ptr[dev] + kPartialFloats, 0, kCounterInts * sizeof(int));
}
}  // namespace rq

extern "C" int rq_decode_attn_noalloc(rq_cache *cache, int layer, int loop, const void *q_bf16, float *out,
                                      float softmax_scale, void *stream) {
    if (!cache || !q_bf16 || !out) return RQ_ERR_INVALID;
    // the scratch address is per device: the current device must be the cache's
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return RQ_ERR_CUDA;
    }
    if (dev != rq::cache_device(cache)) return RQ_ERR_INVALID;
    float *scratch = nullptr;
    const int st = scratch_for_current_device(&scratch);
    if (st != RQ_OK) return st;
    return rq::decode_with_scratch(cache, layer, loop, q_bf16, out, softmax_scale, stream, scratch, kPartialFloats,
                                   reinterpret_cast<int *>(scratch + kPartialFloats), kCounterInts);
}
