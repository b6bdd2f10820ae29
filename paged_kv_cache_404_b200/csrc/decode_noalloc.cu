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
// symbol), so its address is looked up once per device with
// cudaGetSymbolAddress, with that device current, on the first call made on
// that device, and cached.
#include "pagedkv.h"
#include "pkv_common.cuh"

// The scratch itself.  Nothing in it has to start at zero: every decode call
// begins with its plan kernel, which rewrites the header (work counter, unit
// count, partition size) and the work list before any other kernel reads them,
// and partials are written before they are read.
static __device__ __align__(256) unsigned char g_decode_scratch[PKV_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;

// Device address of g_decode_scratch per device ordinal (null until the first
// call on that device).  Two host threads racing on the first call store the
// same value.
void* g_scratch_address[kMaxDevices];

}  // namespace

extern "C" int pkv_paged_attention_decode_noalloc(void* out, const void* q, int q_dtype, const void* k_pool,
                                                  const void* v_pool, int cache_dtype, const int32_t* block_tables,
                                                  int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                                                  int max_context_len, int num_blocks, int block_size, int num_heads,
                                                  int num_kv_heads, int head_dim, float scale, float k_scale,
                                                  float v_scale, int partition_tokens, int32_t* err_count,
                                                  void* stream) {
    // Bounds first: a problem whose scratch would not fit is refused before any CUDA call.
    const size_t need =
        pkv_decode_workspace_bytes(num_seqs, num_heads, head_dim, max_context_len, partition_tokens);
    if (need == 0 || need > (size_t)PKV_NOALLOC_SCRATCH_BYTES) return PKV_EINVAL;

    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ECUDA;
    if (dev < 0 || dev >= kMaxDevices) return PKV_EUNSUPPORTED;
    void* scratch = g_scratch_address[dev];
    if (scratch == nullptr) {
        if (cudaGetSymbolAddress(&scratch, g_decode_scratch) != cudaSuccess || scratch == nullptr)
            return PKV_ECUDA;
        g_scratch_address[dev] = scratch;
    }
    return pkv_paged_attention_decode(out, q, q_dtype, k_pool, v_pool, cache_dtype, block_tables,
                                      max_blocks_per_seq, context_lens, num_seqs, max_context_len, num_blocks,
                                      block_size, num_heads, num_kv_heads, head_dim, scale, k_scale, v_scale,
                                      partition_tokens, scratch, (size_t)PKV_NOALLOC_SCRATCH_BYTES, err_count,
                                      stream);
}
