// select_static.cu -- tri_select_topB_static: the top-B selection with its
// scratch memory in a statically allocated device array, for callers that
// cannot allocate device memory.
//
// Some callers of this library cannot provide a workspace: a serving engine
// whose memory manager owns every byte of device memory and hands a plugin
// only its input and output tensors, or a latency-critical path where calling
// cudaMalloc (which can synchronise the device and can fail under memory
// pressure) is not allowed.  For them this entry point keeps the selection's
// scratch (radix histograms and per-chunk counts) in the file-scope array
// below, which every GPU that loads the library reserves until the process
// exits.  It runs exactly the kernels of tri_select_topB, so its results are
// identical.
#include <mutex>

#include "tri_internal.cuh"
#include "tri_launch.h"

namespace {

// 1 MiB: enough for e.g. 40 units of up to 131072 keys, or 42 units of 32768.
constexpr size_t kStaticScratchBytes = size_t(1) << 20;

static __device__ __align__(256) uint8_t g_select_scratch[kStaticScratchBytes];

// Device address of g_select_scratch on the current device.  Looked up with
// that device current on every call made outside stream capture (so a
// context re-created after cudaDeviceReset is followed), and remembered per
// device for calls made while the stream is being captured, which must come
// after one uncaptured call on that device.
tri_status scratch_address(cudaStream_t s, void** out) {
    static std::mutex mu;
    static void* addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TRI_ERR_CUDA;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return TRI_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (cs == cudaStreamCaptureStatusNone) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || !p) return TRI_ERR_CUDA;
        addr[dev] = p;
    } else if (!addr[dev]) {
        return TRI_ERR_CUDA;  // first call on this device under capture
    }
    *out = addr[dev];
    return TRI_OK;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3) == 0; }

}  // namespace

extern "C" size_t tri_select_static_scratch_bytes(void) { return kStaticScratchBytes; }

extern "C" tri_status tri_select_topB_static(const float* final_score, int64_t n_units,
                                             int64_t cap, const int32_t* n_valid, int64_t B,
                                             int32_t* kept_idx, int32_t* n_kept, void* stream) {
    if (!final_score || !kept_idx || !n_kept || n_units < 1 || cap < 1 || B < 1)
        return TRI_ERR_INVALID_ARG;
    if (B > INT32_MAX || n_units > 65535 || cap > (int64_t(1) << 30)) return TRI_ERR_UNSUPPORTED;
    if (!aligned4(final_score) || !aligned4(kept_idx) || !aligned4(n_kept) ||
        (n_valid && !aligned4(n_valid)))
        return TRI_ERR_INVALID_ARG;
    tri::begin_launches();
    // The layout of tri_select_topB's workspace: flag word, three radix
    // histograms per unit, per-chunk counts.
    const tri::SelectWs lay = tri::select_ws(tri::kWsHeader, n_units, cap);
    if (lay.total > kStaticScratchBytes) return TRI_ERR_SCRATCH_LIMIT;
    const size_t hists = lay.hists, counts = lay.counts;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    void* ws = nullptr;
    const tri_status st = scratch_address(s, &ws);
    if (st != TRI_OK) return st;
    char* base = static_cast<char*>(ws);
    // The histograms accumulate with atomics: zero them (and the flag word).
    if (cudaMemsetAsync(base, 0, counts, s) != cudaSuccess) return TRI_ERR_CUDA;
    uint32_t* h = reinterpret_cast<uint32_t*>(base + hists);
    uint32_t* flag = reinterpret_cast<uint32_t*>(base);
    for (int p = 0; p < 3; ++p)
        if (tri::launch_radix_pass(final_score, n_units, cap, n_valid, B, h, p, flag, s) !=
            cudaSuccess)
            return TRI_ERR_CUDA;
    if (tri::launch_select_finish(final_score, n_units, cap, n_valid, B, h,
                                  reinterpret_cast<uint2*>(base + counts), kept_idx, n_kept,
                                  s) != cudaSuccess)
        return TRI_ERR_CUDA;
    return TRI_OK;
}
