// decode_noalloc.cu -- paged decode attention for callers that cannot allocate.
//
// pkv_paged_attention_decode needs scratch (the partition plan, a work counter
// and the split-context partials) that its caller allocates and passes in.
// Some callers cannot allocate device memory where they run the decode: a
// plug-in living inside a host program that owns all device memory (and gives
// its plug-ins no allocator), a loop that must not call cudaMalloc/cudaFree
// because they synchronise the device and stall every stream, a hard
// latency budget that allocation would break, or code running while a CUDA
// graph or a memory pool forbids new allocations.  This entry point gives them
// the same decode with no allocation at all: the scratch is a fixed-size array
// that the library declares in device memory at file scope.
//
// The array costs PKV_NOALLOC_SCRATCH_BYTES of device memory on every GPU that
// loads this library's kernels, held until the process exits.  Host code cannot
// use the array's name as a device address (on the host it is only a stand-in
// symbol), so its address is looked up with cudaGetSymbolAddress, with the
// device current, on the first call made in a device's context, and kept for
// later calls in that same context.  The context is recognised by the driver's
// unique context id, so a context destroyed and created again (cudaDeviceReset,
// for one) gets a fresh lookup instead of a stale address.
#include <cudaTypedefs.h>

#include <mutex>

#include "pagedkv.h"
#include "pkv_common.cuh"

// The scratch itself.  Nothing in it has to start at zero: every decode call
// begins with its plan kernel, which rewrites the header (work counter, unit
// count, partition size) and the work list before any other kernel reads them,
// and partials are written before they are read.
static __device__ __align__(256) unsigned char g_decode_scratch[PKV_NOALLOC_SCRATCH_BYTES];

namespace pkv {
int decode_check_args(const void* out, const void* q, int q_dtype, const void* k_pool, const void* v_pool,
                      int cache_dtype, const int32_t* block_tables, int max_blocks_per_seq,
                      const int32_t* context_lens, int num_seqs, int max_context_len, int num_blocks, int block_size,
                      int num_heads, int num_kv_heads, int head_dim, float k_scale, float v_scale,
                      int partition_tokens, const int32_t* err_count);
}  // namespace pkv

namespace {

constexpr int kMaxDevices = 64;

// The scratch's device address per device ordinal, with the id of the context
// it was looked up in (address null: not looked up yet).  Guarded by g_mutex.
struct ScratchSlot {
    unsigned long long ctx_id;
    void* addr;
};
ScratchSlot g_slots[kMaxDevices];
std::mutex g_mutex;

// Unique id of the calling thread's current context; false if there is none
// or the driver does not say.
bool current_context_id(unsigned long long* id) {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static bool looked_up = false;
    if (!looked_up) {  // under g_mutex
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
        fn = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
        looked_up = true;
    }
    if (get_current == nullptr || get_id == nullptr) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_decode_scratch in the current device's context.
int scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ECUDA;
    if (dev < 0 || dev >= kMaxDevices) return PKV_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    unsigned long long id = 0;
    if (current_context_id(&id) && g_slots[dev].addr != nullptr && g_slots[dev].ctx_id == id) {
        *out = g_slots[dev].addr;
        return PKV_OK;
    }
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_decode_scratch) != cudaSuccess || addr == nullptr) return PKV_ECUDA;
    // the lookup made the device's context current if it was not; keep the
    // address only if that context can be recognised on later calls
    if (current_context_id(&id)) {
        g_slots[dev].ctx_id = id;
        g_slots[dev].addr = addr;
    } else {
        g_slots[dev].addr = nullptr;
    }
    *out = addr;
    return PKV_OK;
}

}  // namespace

extern "C" int pkv_paged_attention_decode_noalloc(void* out, const void* q, int q_dtype, const void* k_pool,
                                                  const void* v_pool, int cache_dtype, const int32_t* block_tables,
                                                  int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                                                  int max_context_len, int num_blocks, int block_size, int num_heads,
                                                  int num_kv_heads, int head_dim, float scale, float k_scale,
                                                  float v_scale, int partition_tokens, int32_t* err_count,
                                                  void* stream) {
    // The decode's own argument checks first (same statuses as the workspace
    // entry point), then the bound: a problem whose scratch would not fit is
    // refused before any CUDA call.
    const int st = pkv::decode_check_args(out, q, q_dtype, k_pool, v_pool, cache_dtype, block_tables,
                                          max_blocks_per_seq, context_lens, num_seqs, max_context_len, num_blocks,
                                          block_size, num_heads, num_kv_heads, head_dim, k_scale, v_scale,
                                          partition_tokens, err_count);
    if (st != PKV_OK || num_seqs == 0) return st;
    const size_t need =
        pkv_decode_workspace_bytes(num_seqs, num_heads, head_dim, max_context_len, partition_tokens);
    if (need == 0 || need > (size_t)PKV_NOALLOC_SCRATCH_BYTES) return PKV_EINVAL;

    void* scratch = nullptr;
    const int sa = scratch_address(&scratch);
    if (sa != PKV_OK) return sa;
    return pkv_paged_attention_decode(out, q, q_dtype, k_pool, v_pool, cache_dtype, block_tables,
                                      max_blocks_per_seq, context_lens, num_seqs, max_context_len, num_blocks,
                                      block_size, num_heads, num_kv_heads, head_dim, scale, k_scale, v_scale,
                                      partition_tokens, scratch, (size_t)PKV_NOALLOC_SCRATCH_BYTES, err_count,
                                      stream);
}
