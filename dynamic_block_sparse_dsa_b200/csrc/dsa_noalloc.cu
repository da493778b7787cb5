// dsa_noalloc.cu -- decode attention for callers that cannot allocate.
//
// Some callers cannot call cudaMalloc at all: an engine plugin whose enqueue
// path must neither allocate nor synchronise, a runtime that hands out all
// device memory from an allocator it owns, or code that runs where a failed
// allocation cannot be recovered from.  cudaMalloc may synchronise the device
// and may fail under memory pressure, so such callers cannot provide the
// split-KV workspace that dsa_sparse_attn_decode asks for.
//
// dsa_sparse_attn_decode_noalloc keeps that scratch in a fixed array in this
// library's own device memory instead: a file-scope __device__ array of
// DSA_NOALLOC_SCRATCH_BYTES (16 MiB) that every GPU which loads the library
// holds until the process exits.  The caller still passes inputs and outputs.
// The array's name is only a host-side stand-in in host code, so the first
// call on each device (with that device current) looks up its device address
// with cudaGetSymbolAddress and caches it; that first call should therefore
// come before any stream capture.  The cached address belongs to the device's
// primary context: after cudaDeviceReset (or any reset of that context) the
// module is loaded again and the cached address is stale, so a process that
// resets a device must not call this entry point on it afterwards.
// Every argument is checked on the host before anything is enqueued: a call
// that is refused (bad sizes, a problem too large for the scratch) leaves the
// scratch untouched.  Every call zeroes the split counters the
// kernel relies on, then runs the same split-KV decode as
// dsa_sparse_attn_decode on that scratch.  All calls share the one array, so
// calls whose work overlaps on the GPU (other streams, other threads) race
// and must be serialised by the caller.  No cudaMalloc, cudaFree or other
// allocating routine is called.
#include <mutex>

#include "dsa_kernels.h"

namespace {

constexpr size_t kScratchBytes = DSA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

// device address of the scratch array on the current device (looked up once)
int scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DSA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return DSA_OK;
}

}  // namespace

extern "C" int dsa_sparse_attn_decode_noalloc(const dsa_kv_cache *cache, const dsa_seqs *seqs,
                                              const dsa_queries *queries, const void *q, int32_t num_q_heads,
                                              const int32_t *sel, const int32_t *cnt, int32_t k_max,
                                              float sm_scale, void *out, float *lse, int32_t *dev_err,
                                              dsa_stream_t stream) {
    // every host-side check of the regular entry first: nothing below may
    // touch the device for a call that entry would refuse
    int rc = dsa::check_decode_attn_args(cache, seqs, queries, q, num_q_heads, sel, cnt, k_max, sm_scale, out, lse);
    if (rc != DSA_OK) return rc;
    if (queries->total_q == 0) return DSA_OK;
    const size_t need =
        dsa_sparse_attn_decode_workspace_size(queries->total_q, num_q_heads, cache->num_kv_heads, k_max);
    if (need == 0) return DSA_ERR_INVALID_ARG;
    if (need > kScratchBytes) return DSA_ERR_WORKSPACE;   // problem too large for the fixed scratch
    // the decode workspace starts with one int32 split counter per (query, KV
    // head); they must read zero when the kernel starts
    const size_t counter_bytes = (size_t)queries->total_q * cache->num_kv_heads * sizeof(int32_t);
    if (counter_bytes > need) return DSA_ERR_INVALID_ARG;
    void *scratch = nullptr;
    rc = scratch_address(&scratch);
    if (rc != DSA_OK) return rc;
    if (cudaMemsetAsync(scratch, 0, counter_bytes, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return DSA_ERR_CUDA;
    return dsa_sparse_attn_decode(cache, seqs, queries, q, num_q_heads, sel, cnt, k_max, sm_scale, out, lse,
                                  scratch, kScratchBytes, dev_err, stream);
}
