// Decode attention for callers that cannot allocate device memory.
//
// Some callers have no way to allocate device memory for a workspace: code
// that runs inside an engine which reserves all device memory for its own
// pool and forbids other allocations, plug-ins handed only the tensors of one
// call, or latency-critical paths where a cudaMalloc (which can block and
// synchronize the device) is not acceptable.  tq_decode_attn_noalloc serves
// them: it runs exactly tq_decode_attn, but its scratch is a file-scope
// device array that is part of this library's module image.
#include <mutex>

#include <cuda_runtime.h>

#include "tq_internal.h"

namespace {

// One copy per device that loads the library; it lives until the process
// exits.  All calls on a device share it.
static __device__ __align__(256) uint8_t g_noalloc_scratch[TQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
void *g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// In host code `g_noalloc_scratch` names a host-side stand-in, not device
// memory: the device address must be looked up, once per device, with that
// device current.
int scratch_of_current_device(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ECUDA;
    if (dev < 0 || dev >= kMaxDevices) return TQ_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return TQ_ECUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return TQ_OK;
}

}  // namespace

extern "C" int tq_decode_attn_noalloc(const tq_params *kp, const tq_params *vp, const tq_cache_desc *desc,
                                      const void *Q, int B, int Hq, const int32_t *block_table, int max_blocks,
                                      const int32_t *seq_lens, int max_seq_len, const void *cache,
                                      int64_t num_blocks, void *out, float *lse, float *logits,
                                      int64_t logits_stride, void *stream) {
    const size_t need = tq_decode_workspace_bytes(desc, B, Hq, max_seq_len);
    if (need == 0) return TQ_EINVAL;
    if (need > size_t(TQ_NOALLOC_SCRATCH_BYTES)) return TQ_ESCRATCH;
    void *ws = nullptr;
    const int st = scratch_of_current_device(&ws);
    if (st != TQ_OK) return st;
    // The header holds the device status word, which kernels only OR into:
    // clear it so flags from an earlier call do not carry over.
    if (cudaMemsetAsync(ws, 0, tq::kWsHeader, static_cast<cudaStream_t>(stream)) != cudaSuccess) return TQ_ECUDA;
    return tq_decode_attn(kp, vp, desc, Q, B, Hq, block_table, max_blocks, seq_lens, max_seq_len, cache,
                          num_blocks, out, lse, logits, logits_stride, ws, size_t(TQ_NOALLOC_SCRATCH_BYTES), stream);
}

extern "C" int tq_noalloc_read_status(void *stream, uint32_t *flags) {
    if (!flags) return TQ_EINVAL;
    void *ws = nullptr;
    const int st = scratch_of_current_device(&ws);
    if (st != TQ_OK) return st;
    // the status word sits at the start of the static array's header
    return tq_read_status(ws, stream, flags);
}
