// decode_merge.cu -- log-sum-exp merge of split-context partitions.
//
// A long context is cut into partitions (FlashAttention-2 parallelises over
// the context; iplexlaw.co.kr, section on technical differences); partition p
// of (sequence, query head) left (m_p, l_p, o_p): the max of its base-2 scores,
// the sum of 2^(s - m_p) and its normalised output.  The merge is
//   M = max_p m_p over partitions with l_p > 0,  w_p = l_p 2^(m_p - M),
//   out = sum_p w_p o_p / sum_p w_p,
// and a sequence with a single partition was written by the decode kernel.
//
// One warp per (sequence, query head).  Lanes are 4 partition groups x 8
// head_dim slices (16 elements each): group r takes partitions r, r+4, ...;
// the first 4 x KR partitions are loaded in one round (weights and outputs
// together, before the max is known), so up to 4 x KR partitions cost two
// dependent rounds of loads (the partition count, then the partials); the four
// groups are combined with shuffles at the end.  KR = 4 for a merge of up to 32
// warps per SM, KR = 2 above (measured on B200, 148 SMs: KR = 4 took 3-6 us off the
// calls with 2,048 and 4,096 merge warps; at 6,144 and 16,384 warps KR = 2 was as
// fast or faster, where more resident warps hide the latency better than more
// loads per warp).  Deterministic: the order of additions depends only on the
// partition count.
#include "pkv_common.cuh"

namespace pkv {

template <int D, int KR, typename OutT>
__global__ void __launch_bounds__(256) decode_merge_kernel(DecodeParams p) {
    pdl_wait();
    constexpr int SL = D / 8;   // head_dim elements per lane
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= p.num_seqs * p.num_heads) return;
    const int s = warp / p.num_heads;
    const int n = p.nparts[s];
    if (n <= 1) return;
    const size_t base = (size_t)warp * p.max_parts;
    const int grp = lane >> 3, slice = lane & 7;

    // The first 4 partitions: each lane group loads its partition's (m, l) and its
    // head_dim slice of its output in one round of loads, before the max is
    // known.  Further partitions take further rounds.
    float M = -INFINITY;
    float2 ml[KR];
    float4 x[KR][SL / 4];
#pragma unroll
    for (int k = 0; k < KR; ++k) {
        const int i = grp + 4 * k;
        ml[k] = make_float2(-INFINITY, 0.f);
        if (i < n) {
            ml[k] = p.part_ml[base + i];
            const float4* src = reinterpret_cast<const float4*>(p.part_o + (base + i) * D + slice * SL);
#pragma unroll
            for (int v = 0; v < SL / 4; ++v) x[k][v] = src[v];
        }
        if (ml[k].y > 0.f) M = fmaxf(M, ml[k].x);
    }
    for (int i = grp + 4 * KR; i < n; i += 4) {
        const float2 m2 = p.part_ml[base + i];
        if (m2.y > 0.f) M = fmaxf(M, m2.x);
    }
    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 8));
    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 16));

    float acc[SL];
#pragma unroll
    for (int e = 0; e < SL; ++e) acc[e] = 0.f;
    float W = 0.f;
    if (M != -INFINITY) {
#pragma unroll
        for (int k = 0; k < KR; ++k) {
            if (grp + 4 * k >= n) continue;
            const float w = ml[k].y > 0.f ? ml[k].y * exp2f(ml[k].x - M) : 0.f;
            W += w;
#pragma unroll
            for (int v = 0; v < SL / 4; ++v) {
                acc[4 * v] += w * x[k][v].x;
                acc[4 * v + 1] += w * x[k][v].y;
                acc[4 * v + 2] += w * x[k][v].z;
                acc[4 * v + 3] += w * x[k][v].w;
            }
        }
        for (int i = grp + 4 * KR; i < n; i += 4) {
            const float2 m2 = p.part_ml[base + i];
            const float w = m2.y > 0.f ? m2.y * exp2f(m2.x - M) : 0.f;
            W += w;
            const float4* src = reinterpret_cast<const float4*>(p.part_o + (base + i) * D + slice * SL);
#pragma unroll
            for (int v = 0; v < SL / 4; ++v) {
                const float4 y = src[v];
                acc[4 * v] += w * y.x;
                acc[4 * v + 1] += w * y.y;
                acc[4 * v + 2] += w * y.z;
                acc[4 * v + 3] += w * y.w;
            }
        }
    }
    // combine the four partition groups (lanes slice, slice+8, slice+16, slice+24)
#pragma unroll
    for (int o = 8; o < 32; o <<= 1) {
        W += __shfl_xor_sync(0xffffffffu, W, o);
#pragma unroll
        for (int e = 0; e < SL; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    }
    if (grp != 0) return;
    const float inv = W > 0.f ? 1.f / W : 0.f;
    OutT* out = static_cast<OutT*>(p.out) + (size_t)warp * D + slice * SL;
    if constexpr (sizeof(OutT) == 4) {
#pragma unroll
        for (int v = 0; v < SL / 4; ++v)
            reinterpret_cast<float4*>(out)[v] =
                make_float4(acc[4 * v] * inv, acc[4 * v + 1] * inv, acc[4 * v + 2] * inv, acc[4 * v + 3] * inv);
    } else {
#pragma unroll
        for (int v = 0; v < SL / 4; ++v) {
            const uint32_t lo = pack_bf16x2(acc[4 * v] * inv, acc[4 * v + 1] * inv);
            const uint32_t hi = pack_bf16x2(acc[4 * v + 2] * inv, acc[4 * v + 3] * inv);
            reinterpret_cast<uint2*>(out)[v] = make_uint2(lo, hi);
        }
    }
}

template <int D, int KR>
cudaError_t launch_merge_kr(const DecodeParams& p, int out_dtype, unsigned grid, cudaStream_t stream) {
    return out_dtype == 0 ? launch_pdl(decode_merge_kernel<D, KR, float>, dim3(grid), dim3(256), 0, stream, p)
                          : launch_pdl(decode_merge_kernel<D, KR, __nv_bfloat16>, dim3(grid), dim3(256), 0, stream, p);
}

// Largest merge, in warps per SM, that takes the KR = 4 form.
constexpr int kMergeWarpsPerSmKr4 = 32;

cudaError_t launch_decode_merge(const DecodeParams& p, int out_dtype, int num_sms, cudaStream_t stream) {
    const long long warps = (long long)p.num_seqs * p.num_heads;
    const unsigned grid = (unsigned)((warps * 32 + 255) / 256);
    const bool kr4 = warps <= (long long)num_sms * kMergeWarpsPerSmKr4;
    if (p.head_dim == 128)
        return kr4 ? launch_merge_kr<128, 4>(p, out_dtype, grid, stream)
                   : launch_merge_kr<128, 2>(p, out_dtype, grid, stream);
    return kr4 ? launch_merge_kr<64, 4>(p, out_dtype, grid, stream) : launch_merge_kr<64, 2>(p, out_dtype, grid, stream);
}

}  // namespace pkv
