// kda_prefill_noalloc: kda_prefill for callers that cannot allocate device
// memory.
//
// Some hosts cannot call cudaMalloc at the point where they run the operator:
// an inference engine that has reserved all device memory for its own pool,
// a real-time loop that cannot take cudaMalloc's implicit synchronisation,
// or a plugin interface that hands over only a stream and tensor pointers.
// This entry point needs no workspace argument: its scratch lives in a
// fixed-size array in this library's device memory, which every GPU that
// loads the library holds until the process exits.
//
// Host code may not pass the array's name to a kernel (on the host it only
// stands for the symbol); the device address is obtained once per device
// with cudaGetSymbolAddress, with that device current, and cached.
#include <mutex>

#include "kda_internal.cuh"

namespace {

// Room for the error word and a sequence-order table of up to
// kNoAllocMaxSeqs sequences (the workspace kda_prefill asks for).
constexpr int kNoAllocMaxSeqs = KDA_NOALLOC_MAX_SEQS;
constexpr size_t kNoAllocBytes = 256 + kNoAllocMaxSeqs * sizeof(int32_t);
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on the
// first call made with that device current).  Returns null on failure.
void *scratch_for_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = ptr;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

namespace kda {
// The array's device address on the current device (null on failure), for
// kda_check_workspace_error(NULL, ...), which reads its error word.
void *noalloc_scratch() { return scratch_for_current_device(); }
}  // namespace kda

extern "C" kda_status kda_prefill_noalloc(const void *q, const void *k, const void *v,
                                          const void *log_alpha, const void *beta,
                                          const float *init_state, const int32_t *cu_seqlens,
                                          int32_t num_seqs, int64_t total_tokens, int32_t H,
                                          int32_t d_k, int32_t d_v, kda_dtype dtype, void *o,
                                          float *final_state, kda_stream_t stream) {
    if (num_seqs > kNoAllocMaxSeqs) return KDA_ERR_UNSUPPORTED;
    // the array holds the workspace of the single-kernel paths (error word and
    // sequence order); kda_prefill takes those paths for a workspace this size
    if (kda::prefill_tc_workspace(num_seqs) > kNoAllocBytes) return KDA_ERR_UNSUPPORTED;
    void *scratch = scratch_for_current_device();
    if (!scratch) return KDA_ERR_CUDA;
    return kda_prefill(q, k, v, log_alpha, beta, init_state, cu_seqlens, num_seqs, total_tokens,
                       H, d_k, d_v, dtype, o, final_state, scratch, kNoAllocBytes, stream);
}
