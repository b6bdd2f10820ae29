// copy_blocks.cu -- whole-block copies: copy-on-write inside a pool, and swap
// between a device pool and a host pool.
//
// Copy-on-write: before a sequence writes into a physical block that other
// sequences still reference, the block is copied and the writer moves to the
// copy (glossary entry "PagedAttention", section "Compartir bloques entre
// secuencias"; iplexlaw.co.kr, "two answers to one request": only the block
// that must split is copied).
//
// Swap: when device memory is full, small pages move to the CPU instead of
// whole sequences, and come back when the sequence runs again ("Le cache KV et
// PagedAttention", gyaansetu.com, "Eviction a granularite fine").  The host pool
// is page-locked memory mapped into the device address space, so the SMs move
// the bytes over the host link directly, block by block, with no staging copy.
//
// A copy moves the whole block (all slots, all heads) in both the K and the V
// pool.  grid.y = pair, grid.z = pool (K or V), grid.x = 16-byte chunks of one
// block in slices of blockDim.x * kUnroll; every load is issued before any store
// so each thread keeps kUnroll 16-byte requests in flight.
#include "pkv_common.cuh"

namespace pkv {

constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4* __restrict__ dst_k, uint4* __restrict__ dst_v,
                                                          const uint4* __restrict__ src_k,
                                                          const uint4* __restrict__ src_v, long long chunks_per_block,
                                                          const int64_t* __restrict__ pairs, int src_blocks,
                                                          int dst_blocks, int32_t* err) {
    pdl_wait();
    pdl_trigger();
    const int pair = blockIdx.y;
    const long long src = pairs[2 * pair];
    const long long dst = pairs[2 * pair + 1];
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
        if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) count_error(err);
        return;
    }
    const uint4* s = (blockIdx.z == 0 ? src_k : src_v) + src * chunks_per_block;
    uint4* d = (blockIdx.z == 0 ? dst_k : dst_v) + dst * chunks_per_block;
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

cudaError_t launch_copy_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v, size_t block_bytes,
                               const int64_t* pairs, int num_pairs, int src_blocks, int dst_blocks, int32_t* err,
                               cudaStream_t stream) {
    const int threads = 256;
    long long chunks = (long long)(block_bytes / 16);
    long long per_cta = (long long)threads * kCopyUnroll;
    dim3 grid((unsigned)((chunks + per_cta - 1) / per_cta), (unsigned)num_pairs, 2);
    return launch_pdl(copy_blocks_kernel, grid, dim3(threads), 0, stream, static_cast<uint4*>(dst_k),
                      static_cast<uint4*>(dst_v), static_cast<const uint4*>(src_k), static_cast<const uint4*>(src_v),
                      chunks, pairs, src_blocks, dst_blocks, err);
}

}  // namespace pkv
