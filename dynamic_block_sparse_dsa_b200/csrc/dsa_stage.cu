// dsa_stage.cu -- host staging of repeated steps: a step's inputs copied in
// from pinned host memory and its results copied back, on two copy streams of
// the library's own, so that the copies of one batch overlap the kernels of
// the others.
//
// Not part of the method the pages describe: runtime plumbing for a loop that
// issues one step per batch from the host (a serving loop).  Every copy is one
// cudaMemcpyAsync; ordering uses one event per slot and direction:
//   in[slot]       the slot's input copies landed        (copy-in stream)
//   consumed[slot] the slot's step ran                   (compute stream)
//   out[slot]      the slot's read-back landed           (copy-out stream)
// begin:  copy-in waits consumed[slot] -> copies -> record in[slot];
//         compute waits in[slot] and out[slot]
// end:    record consumed[slot] on compute; copy-out waits it -> copies ->
//         record out[slot]
#include <cuda_runtime.h>

#include <new>

#include "dsa.h"

struct dsa_stager {
    int device;
    int num_slots;
    cudaStream_t compute, s_in, s_out;
    cudaEvent_t *ev;   // 3 * num_slots: in, consumed, out
    cudaEvent_t join_in, join_out;
};

namespace {
constexpr int kMaxSlots = 4096;
constexpr int kMaxRegions = 64;

int copies(int n, void *const *dst, const void *const *src, const size_t *bytes, cudaMemcpyKind kind,
           cudaStream_t s) {
    for (int i = 0; i < n; ++i) {
        if (bytes[i] == 0) continue;
        if (cudaMemcpyAsync(dst[i], src[i], bytes[i], kind, s) != cudaSuccess) return DSA_ERR_CUDA;
    }
    return DSA_OK;
}

int check_regions(const dsa_stager *st, int32_t slot, int32_t n, void *const *dst, const void *const *src,
                  const size_t *bytes) {
    if (st == nullptr || slot < 0 || slot >= st->num_slots || n < 0 || n > kMaxRegions) return DSA_ERR_INVALID_ARG;
    if (n == 0) return DSA_OK;
    if (dst == nullptr || src == nullptr || bytes == nullptr) return DSA_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i)
        if (bytes[i] != 0 && (dst[i] == nullptr || src[i] == nullptr)) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

void release(dsa_stager *st) {
    if (st->ev != nullptr) {
        for (int i = 0; i < 3 * st->num_slots; ++i)
            if (st->ev[i] != nullptr) cudaEventDestroy(st->ev[i]);
        delete[] st->ev;
    }
    if (st->join_in != nullptr) cudaEventDestroy(st->join_in);
    if (st->join_out != nullptr) cudaEventDestroy(st->join_out);
    if (st->s_in != nullptr) cudaStreamDestroy(st->s_in);
    if (st->s_out != nullptr) cudaStreamDestroy(st->s_out);
    delete st;
}
}  // namespace

extern "C" {

int dsa_stager_create(int32_t num_slots, dsa_stream_t stream, dsa_stager **out) {
    if (out == nullptr) return DSA_ERR_INVALID_ARG;
    *out = nullptr;
    if (num_slots < 1 || num_slots > kMaxSlots) return DSA_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
    dsa_stager *st = new (std::nothrow) dsa_stager{};
    if (st == nullptr) return DSA_ERR_CUDA;
    st->device = dev;
    st->num_slots = num_slots;
    st->compute = reinterpret_cast<cudaStream_t>(stream);
    st->ev = new (std::nothrow) cudaEvent_t[3 * (size_t)num_slots]();
    bool ok = st->ev != nullptr &&
              cudaStreamCreateWithFlags(&st->s_in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&st->s_out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&st->join_in, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&st->join_out, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < 3 * num_slots; ++i)
        ok = cudaEventCreateWithFlags(&st->ev[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
        release(st);
        return DSA_ERR_CUDA;
    }
    *out = st;
    return DSA_OK;
}

int dsa_stager_destroy(dsa_stager *st) {
    if (st == nullptr) return DSA_OK;
    // the copy streams may still hold copies: let them finish first
    int rc = DSA_OK;
    if (cudaStreamSynchronize(st->s_in) != cudaSuccess || cudaStreamSynchronize(st->s_out) != cudaSuccess)
        rc = DSA_ERR_CUDA;
    release(st);
    return rc;
}

int dsa_stager_begin(dsa_stager *st, int32_t slot, int32_t n, void *const *dev_dst, const void *const *host_src,
                     const size_t *bytes) {
    int rc = check_regions(st, slot, n, dev_dst, reinterpret_cast<const void *const *>(host_src), bytes);
    if (rc != DSA_OK) return rc;
    cudaEvent_t ev_in = st->ev[3 * slot], ev_consumed = st->ev[3 * slot + 1], ev_out = st->ev[3 * slot + 2];
    // the device inputs are still read by the slot's previous step until it has run
    if (cudaStreamWaitEvent(st->s_in, ev_consumed, 0) != cudaSuccess) return DSA_ERR_CUDA;
    rc = copies(n, dev_dst, host_src, bytes, cudaMemcpyHostToDevice, st->s_in);
    if (rc != DSA_OK) return rc;
    if (cudaEventRecord(ev_in, st->s_in) != cudaSuccess) return DSA_ERR_CUDA;
    // the step reads the new inputs and overwrites outputs the previous read-back copies
    if (cudaStreamWaitEvent(st->compute, ev_in, 0) != cudaSuccess ||
        cudaStreamWaitEvent(st->compute, ev_out, 0) != cudaSuccess)
        return DSA_ERR_CUDA;
    return DSA_OK;
}

int dsa_stager_end(dsa_stager *st, int32_t slot, int32_t n, void *const *host_dst, const void *const *dev_src,
                   const size_t *bytes) {
    int rc = check_regions(st, slot, n, host_dst, dev_src, bytes);
    if (rc != DSA_OK) return rc;
    cudaEvent_t ev_consumed = st->ev[3 * slot + 1], ev_out = st->ev[3 * slot + 2];
    if (cudaEventRecord(ev_consumed, st->compute) != cudaSuccess ||
        cudaStreamWaitEvent(st->s_out, ev_consumed, 0) != cudaSuccess)
        return DSA_ERR_CUDA;
    rc = copies(n, host_dst, dev_src, bytes, cudaMemcpyDeviceToHost, st->s_out);
    if (rc != DSA_OK) return rc;
    return cudaEventRecord(ev_out, st->s_out) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

int dsa_stager_wait(dsa_stager *st, int32_t slot) {
    if (st == nullptr || slot < 0 || slot >= st->num_slots) return DSA_ERR_INVALID_ARG;
    return cudaEventSynchronize(st->ev[3 * slot + 2]) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

int dsa_stager_join(dsa_stager *st) {
    if (st == nullptr) return DSA_ERR_INVALID_ARG;
    if (cudaEventRecord(st->join_in, st->s_in) != cudaSuccess ||
        cudaEventRecord(st->join_out, st->s_out) != cudaSuccess ||
        cudaStreamWaitEvent(st->compute, st->join_in, 0) != cudaSuccess ||
        cudaStreamWaitEvent(st->compute, st->join_out, 0) != cudaSuccess)
        return DSA_ERR_CUDA;
    return DSA_OK;
}

}  // extern "C"
