// copy_blocks.cu -- copy-on-write block copy.
//
// Before a sequence writes into a physical block that other sequences still
// reference, the block is copied and the writer moves to the copy (glossary
// entry "PagedAttention", section "Compartir bloques entre secuencias";
// iplexlaw.co.kr, "two answers to one request": only the block that must split
// is copied).  A copy moves the whole block (all slots, all heads) in both the
// K and the V pool.
//
// HBM-bound: grid.y = pair, grid.z = pool (K or V), grid.x = 16-byte chunks of
// one block in slices of blockDim.x * kUnroll; every load is issued before any
// store so each thread keeps kUnroll 16-byte requests in flight.
#include "pkv_common.cuh"

namespace pkv {

constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                                                          long long chunks_per_block,
                                                          const int64_t* __restrict__ pairs, int num_blocks,
                                                          int32_t* err) {
    pdl_wait();
    pdl_trigger();
    const int pair = blockIdx.y;
    const long long src = pairs[2 * pair];
    const long long dst = pairs[2 * pair + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) count_error(err);
        return;
    }
    uint4* pool = blockIdx.z == 0 ? k_pool : v_pool;
    const uint4* s = pool + src * chunks_per_block;
    uint4* d = pool + dst * chunks_per_block;
    const long long base = (long long)blockIdx.x * blockDim.x * kCopyUnroll + threadIdx.x;
    uint4 r[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        long long c = base + (long long)u * blockDim.x;
        if (c < chunks_per_block) r[u] = __ldcs(s + c);
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        long long c = base + (long long)u * blockDim.x;
        if (c < chunks_per_block) __stcs(d + c, r[u]);
    }
}

cudaError_t launch_copy_blocks(void* k_pool, void* v_pool, size_t block_bytes, const int64_t* pairs,
                               int num_pairs, int num_blocks, int32_t* err, cudaStream_t stream) {
    const int threads = 256;
    long long chunks = (long long)(block_bytes / 16);
    long long per_cta = (long long)threads * kCopyUnroll;
    dim3 grid((unsigned)((chunks + per_cta - 1) / per_cta), (unsigned)num_pairs, 2);
    return launch_pdl(copy_blocks_kernel, grid, dim3(threads), 0, stream, static_cast<uint4*>(k_pool),
                      static_cast<uint4*>(v_pool), chunks, pairs, num_blocks, err);
}

}  // namespace pkv
