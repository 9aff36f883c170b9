// gpt_lm_head_loss_noalloc: the tied head + cross-entropy with its scratch held in a static
// device array of this library instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they need a loss: a serving
// process that handed all of its GPU memory to a fixed pool when it started, a plugin running
// inside another framework whose allocator it may not go around, or a latency-critical loop
// that cannot afford cudaMalloc's cost and implicit device synchronisation.  This entry point
// lets them compute the head and the loss with nothing but their inputs and outputs.
//
// The scratch is kNoAllocScratchBytes of global memory that every GPU holds from the moment it
// first uses this library until the process exits.  All calls on a device share it and it keeps
// whatever the last call left in it, so two calls whose work overlaps on the GPU (different
// streams, no ordering between them) corrupt each other's partial sums; serialise them.
#include <mutex>

#include "internal.h"

#define GPT_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_lm_head_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_on_device[kMaxDevices] = {nullptr};

// Device address of g_lm_head_scratch on the current device.  In host code the array's name is
// only a stand-in, so the address is looked up once per device with that device current and kept
// for the life of the process (a device reset invalidates it; the header says so).
int scratch_for_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GPT_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GPT_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_on_device[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_lm_head_scratch) != cudaSuccess || !p) return GPT_ERR_CUDA;
        g_scratch_on_device[dev] = p;
    }
    *out = g_scratch_on_device[dev];
    return GPT_OK;
}

}  // namespace

GPT_API int gpt_lm_head_loss_noalloc(const void* u, const void* wte, const int64_t* targets, int rows, int C,
                                     int V, int dtype, void* logits, float* loss, float* row_loss,
                                     double* loss_sum_count, void* stream, int flags) {
    if (rows < 1 || V < 1) return GPT_ERR_BAD_SHAPE;
    if (gpt_lm_head_workspace_bytes(rows, V) > kNoAllocScratchBytes) return GPT_ERR_WS_TOO_SMALL;
    void* scratch = nullptr;
    const int rc = scratch_for_current_device(&scratch);
    if (rc != GPT_OK) return rc;
    // The status word at the start of the scratch is zeroed by the call before any kernel runs;
    // every other byte the kernels read was written earlier in the same call.
    return gpt_lm_head_loss(u, wte, targets, rows, C, V, dtype, logits, loss, row_loss, loss_sum_count, scratch,
                            kNoAllocScratchBytes, stream, flags);
}
