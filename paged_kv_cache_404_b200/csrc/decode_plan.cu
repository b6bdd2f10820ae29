// decode_plan.cu -- partition plan and log-sum-exp merge for split contexts.
//
// Long contexts are cut into partitions of P tokens so that every SM has work
// (FlashAttention-2 parallelises over the context, iplexlaw.co.kr, section on
// technical differences).  Each partition yields (m, l, o): running max of the
// base-2 scores, sum of 2^(s - m), and the normalised output.  Partitions are
// merged with weights l_p * 2^(m_p - M), M = max_p m_p.
//
// The plan runs on the device because the context lengths live there: one CTA
// picks P from the actual lengths, then writes a work list of (sequence,
// partition) items ordered by size, largest first (full partitions, then the
// tails by decreasing length), so that a persistent kernel handing out items
// through an atomic counter finishes with small items (longest processing
// time first).
#include "pkv_common.cuh"

namespace pkv {

constexpr int kPlanThreads = 1024;
constexpr int kMaxBuckets = 1024;

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

__device__ __forceinline__ int bucket_of(int nblk, int nb_top, int nbuckets) {
    // bucket 0 = one block ... nbuckets-1 = a full partition
    return (int)(((long long)(nblk - 1) * nbuckets) / nb_top);
}

__global__ void __launch_bounds__(kPlanThreads) decode_plan_kernel(DecodeParams p, int fixed_partition, int min_partition,
                                                                   int num_candidates, int target_units,
                                                                   int zero_out_dtype) {
    __shared__ int hist[kMaxBuckets];
    __shared__ unsigned long long red[kPlanThreads / 32];
    __shared__ int chosen;
    const int tid = threadIdx.x;

    // 1. partition size
    if (fixed_partition > 0) {
        if (tid == 0) chosen = fixed_partition;
    } else {
        if (tid == 0) chosen = min_partition;
        // largest candidate (min_partition << c) that still yields target_units units
        for (int c = num_candidates - 1; c >= 0; --c) {
            const int P = min_partition << c;
            unsigned long long units = 0;
            for (int s = tid; s < p.num_seqs; s += kPlanThreads)
                units += (unsigned long long)ceil_div(clamped_len(p, s, false), P);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) units += __shfl_xor_sync(0xffffffffu, units, o);
            if ((tid & 31) == 0) red[tid >> 5] = units;
            __syncthreads();
            if (tid < 32) {
                unsigned long long u = red[tid];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) u += __shfl_xor_sync(0xffffffffu, u, o);
                if (tid == 0 && u * (unsigned long long)p.num_kv_heads >= (unsigned long long)target_units &&
                    chosen == min_partition)
                    chosen = P;
            }
            __syncthreads();
            if (chosen != min_partition) break;
        }
    }
    __syncthreads();
    const int P = chosen;
    const int nb_top = P / kBlockSize;
    const int nbuckets = nb_top < kMaxBuckets ? nb_top : kMaxBuckets;

    // 2. histogram of item sizes
    for (int b = tid; b < kMaxBuckets; b += kPlanThreads) hist[b] = 0;
    __syncthreads();
    for (int s = tid; s < p.num_seqs; s += kPlanThreads) {
        const int L = clamped_len(p, s, true);
        const int nfull = L / P, tail = L - nfull * P;
        p.nparts[s] = nfull + (tail > 0);
        if (nfull) atomicAdd(&hist[nbuckets - 1], nfull);
        if (tail) atomicAdd(&hist[bucket_of(ceil_div(tail, kBlockSize), nb_top, nbuckets)], 1);
        if (L == 0) {
            // an empty context produces a zero output row (nothing else writes it)
            const size_t row = (size_t)s * p.num_heads * p.head_dim;
            const int n = p.num_heads * p.head_dim;
            for (int e = 0; e < n; ++e) {
                if (zero_out_dtype == 0)
                    static_cast<float*>(p.out)[row + e] = 0.f;
                else
                    static_cast<__nv_bfloat16*>(p.out)[row + e] = __float2bfloat16(0.f);
            }
        }
    }
    __syncthreads();

    // 3. exclusive scan, largest bucket first (serial over <= 1024 buckets by one warp)
    if (tid < 32) {
        int running = 0;
        for (int base = nbuckets - 1; base >= 0; base -= 32) {
            const int b = base - tid;
            int v = b >= 0 ? hist[b] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (tid >= o) incl += n;
            }
            if (b >= 0) hist[b] = running + incl - v;
            running += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (tid == 0) {
            p.hdr->num_items = running;
            p.hdr->num_units = running * p.num_kv_heads;
            p.hdr->partition = P;
            p.hdr->counter = 0;
            p.hdr->timeout = 0;
        }
    }
    __syncthreads();

    // 4. scatter the items (order inside a bucket does not affect results)
    int2* items = p.items;
    for (int s = tid; s < p.num_seqs; s += kPlanThreads) {
        const int L = clamped_len(p, s, false);
        const int nfull = L / P, tail = L - nfull * P;
        if (nfull) {
            const int base = atomicAdd(&hist[nbuckets - 1], nfull);
            for (int j = 0; j < nfull; ++j) items[base + j] = make_int2(s, j);
        }
        if (tail) {
            const int pos = atomicAdd(&hist[bucket_of(ceil_div(tail, kBlockSize), nb_top, nbuckets)], 1);
            items[pos] = make_int2(s, nfull);
        }
    }
}

// One warp per (sequence, query head): merge the partitions of a split context.
template <int D, typename OutT>
__global__ void __launch_bounds__(256) decode_merge_kernel(DecodeParams p) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= p.num_seqs * p.num_heads) return;
    const int s = warp / p.num_heads;
    const int n = p.nparts[s];
    if (n <= 1) return;  // written directly by the decode kernel (or zero length)
    const size_t base = (size_t)warp * p.max_parts;
    constexpr int E = D / 32;  // elements per lane
    float M = -INFINITY;
    for (int i = lane; i < n; i += 32) {
        float2 ml = p.part_ml[base + i];
        if (ml.y > 0.f) M = fmaxf(M, ml.x);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    float W = 0.f;
    if (M != -INFINITY) {
        for (int i = 0; i < n; ++i) {
            const float2 ml = p.part_ml[base + i];
            if (!(ml.y > 0.f)) continue;
            const float w = ml.y * exp2f(ml.x - M);
            W += w;
            const float* o = p.part_o + (base + i) * D + lane * E;
            if constexpr (E == 4) {
                float4 v = *reinterpret_cast<const float4*>(o);
                acc[0] += w * v.x;
                acc[1] += w * v.y;
                acc[2] += w * v.z;
                acc[3] += w * v.w;
            } else {
#pragma unroll
                for (int e = 0; e < E; ++e) acc[e] += w * o[e];
            }
        }
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    OutT* out = static_cast<OutT*>(p.out) + (size_t)warp * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        if constexpr (sizeof(OutT) == 4)
            out[e] = acc[e] * inv;
        else
            out[e] = __float2bfloat16(acc[e] * inv);
    }
}

cudaError_t launch_decode_plan(const DecodeParams& p, int fixed_partition, int min_partition, int num_candidates,
                               int target_units, int out_dtype, cudaStream_t stream) {
    decode_plan_kernel<<<1, kPlanThreads, 0, stream>>>(p, fixed_partition, min_partition, num_candidates,
                                                        target_units, out_dtype);
    return cudaGetLastError();
}

cudaError_t launch_decode_merge(const DecodeParams& p, int out_dtype, cudaStream_t stream) {
    const int warps = p.num_seqs * p.num_heads;
    const int threads = 256;
    const unsigned grid = (unsigned)((warps * 32 + threads - 1) / threads);
    if (p.head_dim == 128) {
        if (out_dtype == 0)
            decode_merge_kernel<128, float><<<grid, threads, 0, stream>>>(p);
        else
            decode_merge_kernel<128, __nv_bfloat16><<<grid, threads, 0, stream>>>(p);
    } else {
        if (out_dtype == 0)
            decode_merge_kernel<64, float><<<grid, threads, 0, stream>>>(p);
        else
            decode_merge_kernel<64, __nv_bfloat16><<<grid, threads, 0, stream>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace pkv
