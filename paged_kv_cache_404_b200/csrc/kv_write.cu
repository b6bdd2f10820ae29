// kv_write.cu -- KV append: scatter the K and V of new tokens into their slots.
//
// PagedAttention stores token `pos` of a request at row
// (block_table[pos / block_size], pos % block_size) of a shared pool; the
// caller passes that row as a slot (glossary entry "PagedAttention", worked
// example).  A generation step appends only the new token's K and V ("Le cache
// KV et PagedAttention", section "Qu'est-ce que le KV Cache ?").  With an FP8
// cache the value stored is E4M3(x / scale) (glossary entry, "Tecnicas
// relacionadas": FP8 KV cache).
//
// Layout: source [T][Hkv*D]; destination pool rows [NB*16][Hkv*D], so one
// token's K (or V) is one contiguous row of Hkv*D elements.  HBM-bound: each
// thread moves 16 source bytes with vector loads/stores; consecutive threads
// cover consecutive 16-byte chunks of a row, so both sides are coalesced.
#include "pkv_common.cuh"

namespace pkv {

// Same-dtype copy: one 16-byte chunk per thread, for K and V.
__global__ void __launch_bounds__(256) kv_write_copy_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                            const int64_t* __restrict__ slots, int num_tokens,
                                                            uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                                                            long long num_slots, int chunks_per_row,
                                                            int32_t* err) {
    pdl_wait();
    pdl_trigger();
    long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    long long total = (long long)num_tokens * chunks_per_row;
    if (i >= total) return;
    int tok = (int)(i / chunks_per_row);
    int c = (int)(i - (long long)tok * chunks_per_row);
    long long slot = slots[tok];
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (c == 0) count_error(err);
        return;
    }
    size_t dst = (size_t)slot * chunks_per_row + c;
    size_t src = (size_t)tok * chunks_per_row + c;
    uint4 kv = __ldg(k + src);
    uint4 vv = __ldg(v + src);
    k_pool[dst] = kv;
    v_pool[dst] = vv;
}

// E4M3 code of x / scale: IEEE fp32 division rounded to nearest, then
// round-to-nearest-even conversion saturating to +-448.
__device__ __forceinline__ uint32_t quant2(float x0, float x1, float scale) {
    float2 q = make_float2(__fdiv_rn(x0, scale), __fdiv_rn(x1, scale));
    return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3));
}

// bf16/fp32 source -> FP8 cache: each thread produces 16 output codes (16 bytes).
template <typename SrcT>
__global__ void __launch_bounds__(256) kv_write_fp8_kernel(const SrcT* __restrict__ k, const SrcT* __restrict__ v,
                                                           const int64_t* __restrict__ slots, int num_tokens,
                                                           uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                                                           long long num_slots, int chunks_per_row, float k_scale,
                                                           float v_scale, int32_t* err) {
    pdl_wait();
    pdl_trigger();
    long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    long long total = (long long)num_tokens * chunks_per_row;
    if (i >= total) return;
    int tok = (int)(i / chunks_per_row);
    int c = (int)(i - (long long)tok * chunks_per_row);
    long long slot = slots[tok];
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (c == 0) count_error(err);
        return;
    }
    const size_t src = ((size_t)tok * chunks_per_row + c) * 16;  // element index of 16 elements
    const size_t dst = (size_t)slot * chunks_per_row + c;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
        const SrcT* in = (which == 0 ? k : v) + src;
        const float sc = which == 0 ? k_scale : v_scale;
        float x[16];
        if constexpr (sizeof(SrcT) == 2) {
            uint4 a = __ldg(reinterpret_cast<const uint4*>(in));
            uint4 b = __ldg(reinterpret_cast<const uint4*>(in) + 1);
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                x[2 * j] = __uint_as_float(w[j] << 16);
                x[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float4 f = __ldg(reinterpret_cast<const float4*>(in) + j);
                x[4 * j] = f.x;
                x[4 * j + 1] = f.y;
                x[4 * j + 2] = f.z;
                x[4 * j + 3] = f.w;
            }
        }
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t lo = quant2(x[4 * j], x[4 * j + 1], sc);
            uint32_t hi = quant2(x[4 * j + 2], x[4 * j + 3], sc);
            o[j] = lo | (hi << 16);
        }
        (which == 0 ? k_pool : v_pool)[dst] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

cudaError_t launch_kv_write(const void* k, const void* v, int src_dtype, const int64_t* slots, int num_tokens,
                            void* k_pool, void* v_pool, int cache_dtype, long long num_slots, int row_elems,
                            float k_scale, float v_scale, int32_t* err, cudaStream_t stream) {
    // src/cache dtype codes: 0 = f32, 1 = bf16, 2 = fp8
    const int threads = 256;
    if (cache_dtype == src_dtype) {
        int elem = src_dtype == 0 ? 4 : 2;
        int chunks = row_elems * elem / 16;
        long long total = (long long)num_tokens * chunks;
        unsigned grid = (unsigned)((total + threads - 1) / threads);
        return launch_pdl(kv_write_copy_kernel, dim3(grid), dim3(threads), 0, stream, static_cast<const uint4*>(k),
                          static_cast<const uint4*>(v), slots, num_tokens, static_cast<uint4*>(k_pool),
                          static_cast<uint4*>(v_pool), num_slots, chunks, err);
    } else {
        int chunks = row_elems / 16;  // 16 output codes per thread
        long long total = (long long)num_tokens * chunks;
        unsigned grid = (unsigned)((total + threads - 1) / threads);
        if (src_dtype == 1)
            return launch_pdl(kv_write_fp8_kernel<__nv_bfloat16>, dim3(grid), dim3(threads), 0, stream,
                              static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), slots,
                              num_tokens, static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), num_slots, chunks,
                              k_scale, v_scale, err);
        return launch_pdl(kv_write_fp8_kernel<float>, dim3(grid), dim3(threads), 0, stream,
                          static_cast<const float*>(k), static_cast<const float*>(v), slots, num_tokens,
                          static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), num_slots, chunks, k_scale,
                          v_scale, err);
    }
}

}  // namespace pkv
