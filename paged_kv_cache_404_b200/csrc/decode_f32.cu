// decode_f32.cu -- paged decode attention for an fp32 cache (CUDA cores).
//
// Same computation, plan and work units as the tensor-core kernel
// (decode_tc.cu): for each (sequence, partition, kv head) unit, every query
// head of the group attends to the unit's tokens read through the block table
// (glossary entry "PagedAttention", "Como funciona la paginacion"), with an
// online softmax (running max and sum) so no score vector is stored.
// fp32 throughout (no tensor cores: TF32 would not meet fp32 accuracy).  Each
// warp is a persistent worker; lanes split head_dim, so every K and V row is
// one coalesced 256- or 512-byte read and each score is a warp reduction.
#include "pkv_common.cuh"

namespace pkv {

template <int D>
__global__ void __launch_bounds__(256) decode_f32_kernel(const DecodeParams p) {
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31;
    pdl_wait();
    pdl_trigger();
    const int num_units = p.hdr->num_units;
    const float* kpool = static_cast<const float*>(p.k_pool);
    const float* vpool = static_cast<const float*>(p.v_pool);
    for (;;) {
        int u = 0;
        if (lane == 0) u = atomicAdd(&p.hdr->counter, 1);
        u = __shfl_sync(0xffffffffu, u, 0);
        if (u >= num_units) break;
        const int4 item = p.items[u / p.num_kv_heads];
        const int kvh = u % p.num_kv_heads;
        const int s = item.x, part = item.y;
        const int L = clamped_len(p, s, false);
        const int t0 = item.z * kBlockSize, t1 = min(L, t0 + item.w * kBlockSize);
        const int32_t* tab = p.block_tables + (size_t)s * p.max_blocks_per_seq;
        const bool split = p.nparts[s] > 1;
        for (int hh = 0; hh < p.group; ++hh) {
            const int hq = kvh * p.group + hh;
            const float* qrow = static_cast<const float*>(p.q) + ((size_t)s * p.num_heads + hq) * D;
            float q[E], acc[E];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                q[e] = qrow[lane + 32 * e];
                acc[e] = 0.f;
            }
            float m = -INFINITY, l = 0.f;
            for (int tok = t0; tok < t1; ++tok) {
                const int blk = tab[tok / kBlockSize];
                if (blk < 0 || blk >= p.num_blocks) {
                    if (hh == 0 && kvh == 0 && lane == 0 && (tok % kBlockSize == 0)) count_error(p.err);
                    continue;
                }
                const size_t row = (((size_t)blk * kBlockSize + tok % kBlockSize) * p.num_kv_heads + kvh) * D;
                float dot = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) dot += q[e] * kpool[row + lane + 32 * e];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
                const float x = dot * p.score_scale;
                const float mn = fmaxf(m, x);
                const float alpha = exp2f(m - mn);  // m = -inf on the first token: 0
                const float w = exp2f(x - mn);
                l = l * alpha + w;
#pragma unroll
                for (int e = 0; e < E; ++e) acc[e] = acc[e] * alpha + w * vpool[row + lane + 32 * e];
                m = mn;
            }
            const float inv = l > 0.f ? 1.f / l : 0.f;
            if (!split) {
                float* o = static_cast<float*>(p.out) + ((size_t)s * p.num_heads + hq) * D;
#pragma unroll
                for (int e = 0; e < E; ++e) o[lane + 32 * e] = acc[e] * inv;
            } else {
                const size_t slot = ((size_t)s * p.num_heads + hq) * p.max_parts + part;
#pragma unroll
                for (int e = 0; e < E; ++e) p.part_o[slot * D + lane + 32 * e] = acc[e] * inv;
                if (lane == 0) p.part_ml[slot] = make_float2(m, l);
            }
        }
    }
}

cudaError_t launch_decode_f32(const DecodeParams& p, int num_sms, cudaStream_t stream) {
    const int threads = 256;
    const int grid = num_sms * 4;
    if (p.head_dim == 128) return launch_pdl(decode_f32_kernel<128>, dim3(grid), dim3(threads), 0, stream, p);
    return launch_pdl(decode_f32_kernel<64>, dim3(grid), dim3(threads), 0, stream, p);
}

}  // namespace pkv
