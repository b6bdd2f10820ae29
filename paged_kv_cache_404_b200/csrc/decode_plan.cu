// decode_plan.cu -- partition plan and log-sum-exp merge for split contexts.
//
// Long contexts are cut into partitions of P tokens so that every SM has work
// (FlashAttention-2 parallelises over the context, iplexlaw.co.kr, section on
// technical differences).  Each partition yields (m, l, o): running max of the
// base-2 scores, sum of 2^(s - m), and the normalised output.  Partitions are
// merged with weights l_p * 2^(m_p - M), M = max_p m_p.
//
// The merge runs as its own kernel after the decode (decode_merge.cu), so
// that no decode warp sits on a merge's memory latency.
//
// The plan runs on the device because the context lengths live there: one CTA
// picks the partition size from the actual lengths, then writes a work list of
// (sequence, partition, block range) items ordered by size, largest first, so
// that a persistent kernel handing out items through an atomic counter
// finishes with small items (longest processing time first).
#include "pkv_common.cuh"

namespace pkv {

constexpr int kPlanThreads = 1024;  // at most 32 warps: one slot per warp in the candidate counts
constexpr int kMaxBuckets = 128;  // size classes of the longest-first order (a 4-step scan)
constexpr int kMaxCandidates = 12;


__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

__device__ __forceinline__ int bucket_of(int nblk, int nb_top, int nbuckets) {
    // bucket 0 = one block ... nbuckets-1 = a largest partition: (nblk - 1) * nbuckets
    // / nb_top, in 32 bits while the product fits (nbuckets <= 1024, nblk <= nb_top)
    if (nbuckets == nb_top) return nblk - 1;
    if (nb_top < (1 << 21)) return (int)((unsigned)(nblk - 1) * (unsigned)nbuckets / (unsigned)nb_top);
    return (int)(((long long)(nblk - 1) * nbuckets) / nb_top);
}

// Partitions of one sequence of B blocks, in order along the context (the pieces):
//  uniform (user-fixed size): pieces of nb blocks, the last one shorter;
//  geometric (automatic): whole pieces of nb blocks, then the remaining chunk T
//  (1..nb blocks) halved while it exceeds 2*mb: T/2, T/4, ..., then the rest.
//  Each piece is >= mb blocks unless the sequence is shorter, so a sequence of
//  B blocks has at most ceil(B / mb) pieces; under longest-first scheduling the
//  last units handed out are the small ones, which evens out the finish times.
// count_pieces, hist_pieces and scatter_pieces (below) count, histogram and write
// these pieces.

// Shared-prefix groups.  Sequences that start with the same physical blocks
// (parallel samples of one prompt, requests with a common system prompt: the
// glossary entry "PagedAttention", "Compartir bloques entre secuencias") can
// read those blocks once for all of them.  The caller's hints are not trusted:
// here a member is kept only if it is in range and in no group claimed before,
// and the shared count is cut to the blocks every kept member holds in full
// (16 tokens inside its context).  That the members' tables really agree on
// those blocks is checked by the decode kernel, item by item (a subgroup item
// whose members' tables differ is run once per member).  A kept group is split
// into subgroups of at most group_cap members (balanced sizes).  A wrong hint
// costs time, never correctness.
constexpr int kMaxGroupChunks = 32;  // members per group considered: 16 * 32

// One half-warp per group (two groups per warp at a time, so that the loads of
// both groups' three dependent steps -- hint, members, claim -- overlap).
__device__ void build_groups(const DecodeParams& p, int* n_subs, int* n_members) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int half = lane >> 4, hl = lane & 15;
    const int hbase = lane & 16;  // first lane of this half
    for (int s = tid; s < p.num_seqs; s += kPlanThreads) {
        p.seq_sub[s] = -1;
        p.seq_k[s] = 0;
    }
    __syncthreads();
    constexpr int kGroupsPerPass = 2 * (kPlanThreads / 32);
    for (int g0 = 0; g0 < p.num_groups; g0 += kGroupsPerPass) {
        const int gi = g0 + 2 * warp + half;
        int beg = 0, end = 0, k = 0;
        if (gi < p.num_groups) {
            beg = p.group_offsets[gi];
            end = p.group_offsets[gi + 1];
            k = min(p.group_shared_blocks[gi], p.max_blocks_per_seq);
        }
        if (beg < 0 || beg >= p.num_group_seqs) end = beg;  // no members
        end = min(min(end, p.num_group_seqs), beg + 16 * kMaxGroupChunks);
        const bool live = end > beg + 1 && k > 0;
        const int nchunks = live ? (end - beg + 15) >> 4 : 0;
        const int nchunks_warp = max(nchunks, __shfl_xor_sync(0xffffffffu, nchunks, 16));

        // claim the members (bit c of `mine`: member beg + 16c + hl is ours);
        // the length is loaded alongside the claim
        uint32_t mine = 0;
        int count = 0, s_lane = -1;
        for (int c = 0; c < nchunks_warp; ++c) {
            const int i = beg + 16 * c + hl;
            const int s = (c < nchunks && i < end) ? p.group_seqs[i] : -1;
            const bool valid = s >= 0 && s < p.num_seqs;
            const int len = valid ? clamped_len(p, s, false) : 0;
            const bool got = valid && atomicCAS(&p.seq_sub[s], -1, -2) == -1;
            if (got) k = min(k, len / kBlockSize);
            const unsigned b = (__ballot_sync(0xffffffffu, got) >> hbase) & 0xFFFFu;
            if (got) mine |= 1u << c;
            if (c == 0) s_lane = s;
            count += __popc(b);
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) k = min(k, __shfl_xor_sync(0xffffffffu, k, o));

        const bool keep = live && count >= 2 && k > 0;
        const int nsub = keep ? (count + p.group_cap - 1) / p.group_cap : 0;
        int mbase = 0, sbase = 0;
        if (keep && hl == 0) {
            mbase = atomicAdd(n_members, count);
            sbase = atomicAdd(n_subs, nsub);
        }
        mbase = __shfl_sync(0xffffffffu, mbase, hbase);
        sbase = __shfl_sync(0xffffffffu, sbase, hbase);
        if (keep)
            for (int q = hl; q < nsub; q += 16) {
                const int a = (int)(((long long)q * count) / nsub), b = (int)(((long long)(q + 1) * count) / nsub);
                p.sub_info[sbase + q] = make_int4(mbase + a, b - a, k, 0);
            }
        // members in claim order; member of rank r goes to subgroup ((r+1)*nsub - 1) / count
        int rank0 = 0;
        for (int c = 0; c < nchunks_warp; ++c) {
            const bool own = (mine >> c) & 1u;
            const unsigned b = (__ballot_sync(0xffffffffu, own) >> hbase) & 0xFFFFu;
            if (own) {
                const int s = c == 0 ? s_lane : p.group_seqs[beg + 16 * c + hl];
                if (keep) {
                    const int r = rank0 + __popc(b & ((1u << hl) - 1u));
                    p.sub_members[mbase + r] = s;
                    p.seq_sub[s] = sbase + (int)(((long long)(r + 1) * nsub - 1) / count);
                    p.seq_k[s] = k;
                } else {
                    p.seq_sub[s] = -1;  // release
                }
            }
            rank0 += __popc(b);
        }
    }
    __syncthreads();
}

// Halvings of a last chunk of T blocks (T becomes ceil(T / 2) while T > 2 mb):
// ceil(T / 2^k) <= 2 mb first holds at k = ceil(log2(ceil(T / 2 mb))).
__device__ __forceinline__ int halvings(int T, int mb) {
    if (T <= 2 * mb) return 0;
    const unsigned q = ((unsigned)T + 2u * mb - 1u) / (2u * mb);  // >= 2
    return 32 - __clz((int)(q - 1u));
}

// The three helpers below are out of line: each phase of the one-CTA plan runs its
// code once per launch, so its time follows the instructions it fetches more than
// their arithmetic, and one copy serves every call site.
//
// Number of pieces B blocks are cut into (closed form).
__device__ __noinline__ int count_pieces(int B, int nb, int mb, bool geometric) {
    if (B <= 0) return 0;
    if (!geometric) return (B - 1) / nb + 1;
    const int body = (B - 1) / nb;
    return body + 1 + halvings(B - body * nb, mb);
}

// Adds the sizes of the pieces of B blocks to the histogram, the whole pieces
// (all in the top bucket) with one atomic.
__device__ __noinline__ void hist_pieces(int* hist, int B, int nb, int mb, bool geometric, int nbuckets) {
    if (B <= 0) return;
    const int whole = geometric ? (B - 1) / nb : B / nb;
    if (whole > 0) atomicAdd(&hist[nbuckets - 1], whole);
    int T = B - whole * nb;
    if (geometric)
        while (T > 2 * mb) {
            const int piece = T / 2;
            atomicAdd(&hist[bucket_of(piece, nb, nbuckets)], 1);
            T -= piece;
        }
    if (T > 0) atomicAdd(&hist[bucket_of(T, nb, nbuckets)], 1);
}

// Writes the work items of the pieces of B blocks (item.x = code, item.y =
// partition part0, part0 + 1, ... along the context, item.z = first block + k0,
// item.w = blocks), each at the place its bucket's counter in the exclusive-scanned
// histogram gives.  (One atomic per piece measured faster here than one per
// sequence for its whole pieces followed by their stores.)
__device__ __noinline__ void scatter_pieces(int4* items, int* hist, int code, int part0, int k0, int B, int nb,
                                               int mb, bool geometric, int nbuckets) {
    if (B <= 0) return;
    const int whole = geometric ? (B - 1) / nb : B / nb;
    int part = part0, at = 0;
    for (int i = 0; i < whole; ++i, at += nb)
        items[atomicAdd(&hist[nbuckets - 1], 1)] = make_int4(code, part++, k0 + at, nb);
    int T = B - at;
    if (geometric)
        while (T > 2 * mb) {
            const int piece = T / 2;
            items[atomicAdd(&hist[bucket_of(piece, nb, nbuckets)], 1)] = make_int4(code, part++, k0 + at, piece);
            at += piece;
            T -= piece;
        }
    if (T > 0) items[atomicAdd(&hist[bucket_of(T, nb, nbuckets)], 1)] = make_int4(code, part, k0 + at, T);
}

constexpr int kSmemSeqs = 4096;  // per-sequence block counts kept in shared memory up to this many

// Block counts of sequences and subgroups past the shared-memory copies, read from
// global memory.  Out of line: inlined, the compiler (which has seen the same
// addresses loaded in the phase that fills the copies) issues these global reads
// unconditionally beside every shared-memory read and selects afterwards, an L2
// round trip per use.
__device__ __noinline__ int own_blocks_global(const int32_t* lens, const int* seq_k, int cap, int s) {
    const int L = min(max(lens[s], 0), cap);
    return (L + kBlockSize - 1) / kBlockSize - (seq_k != nullptr ? seq_k[s] : 0);
}
__device__ __noinline__ int sub_blocks_global(const int4* sub_info, int q) { return sub_info[q].z; }

__global__ void __launch_bounds__(kPlanThreads) decode_plan_kernel(DecodeParams p, int fixed_partition, int min_partition,
                                                                   int num_candidates, int target_units,
                                                                   int zero_out_dtype) {
    __shared__ int hist[kMaxBuckets];
    __shared__ int own_blocks[kSmemSeqs];  // blocks of sequence s outside its shared prefix
    __shared__ int sub_blocks[kSmemSeqs];  // blocks subgroup q computes for its members
    __shared__ unsigned units_of[kMaxCandidates][32];  // per candidate and warp
    __shared__ int chosen, total_items;
    __shared__ int n_subs, n_members;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // automatic partitioning ends each context with geometrically shrinking pieces
    const bool geometric = fixed_partition == 0;
    const int mb = min_partition / kBlockSize;
    const bool grouped = p.num_groups > 0;

    // The plan reads caller inputs no kernel of this library writes (lengths,
    // tables, group hints) and works in shared memory up to its scan; only its
    // global writes of the header, work list, partition counts and zero rows must
    // wait for the previous kernel on the stream, whose predecessors may still read
    // this workspace and output.  So the wait comes after the scan, and the plan's
    // work overlaps that kernel (the step's KV write).  The grouped plan's member
    // claims and subgroup lists (seq_sub, seq_k, sub_info, sub_members) are written
    // before the wait: the only kernels of this library that let a dependent start
    // early (they signal it right after their own wait) are the KV write, the block
    // copies, the prefill and the decode, and a decode that may still run then is one
    // without prefix groups (a grouped call always ends with the merge, which does
    // not signal early), which never reads those lists; the merge reads only the
    // partition counts and partials.  The wait comes before the plan ends, so the
    // decode that waits for the plan also finds the KV write done.
    pdl_trigger();

    // 0. shared-prefix subgroups: sequence s then owns blocks [seq_k[s], B) and
    //    its subgroup computes blocks [0, seq_k[s]) once for all its members
    if (tid == 0) n_subs = n_members = 0;
    for (int b = tid; b < kMaxBuckets; b += kPlanThreads) hist[b] = 0;
    __syncthreads();
    if (grouped) build_groups(p, &n_subs, &n_members);
    const int num_subs = n_subs;
    // blocks of s after its shared prefix (the length is clamped and counted once, here)
    auto own_of = [&](int s, bool count) {
        return ceil_div(clamped_len(p, s, count), kBlockSize) - (grouped ? p.seq_k[s] : 0);
    };
    for (int s = tid; s < p.num_seqs && s < kSmemSeqs; s += kPlanThreads) own_blocks[s] = own_of(s, true);
    for (int s = kSmemSeqs + tid; s < p.num_seqs; s += kPlanThreads) own_of(s, true);
    for (int q = tid; q < num_subs && q < kSmemSeqs; q += kPlanThreads) sub_blocks[q] = p.sub_info[q].z;
    __syncthreads();
    const int len_cap = min(p.max_blocks_per_seq * kBlockSize, p.max_context_len);
    auto own = [&](int s) {
        return s < kSmemSeqs ? own_blocks[s] : own_blocks_global(p.context_lens, grouped ? p.seq_k : nullptr, len_cap, s);
    };
    auto sub = [&](int q) { return q < kSmemSeqs ? sub_blocks[q] : sub_blocks_global(p.sub_info, q); };

    // 1. largest partition: the largest candidate min_partition << c whose work
    //    list still has target_units units
    if (fixed_partition > 0) {
        if (tid == 0) chosen = fixed_partition;
    } else {
        // per candidate, each warp's count in its own slot (no atomics), summed by one
        // warp; a warp with no sequence and no subgroup writes zeros.  A thread's count is
        // capped at 2^26 so that a warp's sum fits 32 bits (one redux instruction): a cap
        // this far above any target cannot change which candidates reach it.
        const bool busy = tid - lane < p.num_seqs || tid - lane < num_subs;
#pragma unroll 1
        for (int c = 0; c < num_candidates; ++c) {
            unsigned v = 0;
            if (busy) {
                const int nb = (min_partition << c) / kBlockSize;
                unsigned long long n = 0;
                for (int s = tid; s < p.num_seqs; s += kPlanThreads) n += count_pieces(own(s), nb, mb, geometric);
                for (int q = tid; q < num_subs; q += kPlanThreads) n += count_pieces(sub(q), nb, mb, geometric);
                v = __reduce_add_sync(0xffffffffu, (unsigned)min(n, 1ull << 26));
            }
            if (lane == 0) units_of[c][warp] = v;
        }
        __syncthreads();
        if (warp == 0) {
            // with prefix groups, 0.45 of the target: a subgroup's unit carries up to 16
            // score columns, and each further piece costs the plan and the merge
            // (measured on a shared-prefix batch: 101 us with 512-token pieces, 109 with
            // the 256 that the full target leaves)
            const unsigned long long target =
                grouped ? (unsigned long long)target_units * 9 / 20 : (unsigned long long)target_units;
            int P = min_partition;
            for (int c = num_candidates - 1; c >= 0; --c) {
                unsigned long long v = lane < kPlanThreads / 32 ? units_of[c][lane] : 0u;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (v * (unsigned long long)p.num_kv_heads >= target) {
                    P = min_partition << c;
                    break;
                }
            }
            if (lane == 0) chosen = P;
        }
    }
    __syncthreads();
    const int P = chosen;
    const int nb_top = P / kBlockSize;
    const int nbuckets = nb_top < kMaxBuckets ? nb_top : kMaxBuckets;

    // 2. histogram of item sizes
    for (int s = tid; s < p.num_seqs; s += kPlanThreads) hist_pieces(hist, own(s), nb_top, mb, geometric, nbuckets);
    for (int q = tid; q < num_subs; q += kPlanThreads) hist_pieces(hist, sub(q), nb_top, mb, geometric, nbuckets);
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
        if (tid == 0) total_items = running;
    }
    pdl_wait();
    __syncthreads();

    // 4. global writes: header, partitions per sequence (shared ones first), zero
    //    rows of empty contexts, and the items scattered into the work list (order
    //    inside a bucket does not affect results; a sequence's shared partitions
    //    come first, then its own)
    if (tid == 0) {
        p.hdr->num_items = total_items;
        p.hdr->num_units = total_items * p.num_kv_heads;
        p.hdr->partition = P;
        p.hdr->counter = 0;
        p.hdr->timeout = 0;
        p.hdr->num_subs = num_subs;
        p.hdr->num_members = n_members;
    }
    for (int s = tid; s < p.num_seqs; s += kPlanThreads) {
        const int k = grouped ? p.seq_k[s] : 0;
        const int B = own(s);
        const int part = count_pieces(k, nb_top, mb, geometric);
        p.nparts[s] = part + count_pieces(B, nb_top, mb, geometric);
        if (B + k == 0) {
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
        scatter_pieces(p.items, hist, s, part, k, B, nb_top, mb, geometric, nbuckets);
    }
    // subgroup items carry -(subgroup + 1) in place of the sequence
    for (int q = tid; q < num_subs; q += kPlanThreads)
        scatter_pieces(p.items, hist, -(q + 1), 0, 0, sub(q), nb_top, mb, geometric, nbuckets);
}

cudaError_t launch_decode_plan(const DecodeParams& p, int fixed_partition, int min_partition, int num_candidates,
                               int target_units, int out_dtype, cudaStream_t stream) {
    return launch_pdl(decode_plan_kernel, dim3(1), dim3(kPlanThreads), 0, stream, p, fixed_partition, min_partition,
                      num_candidates, target_units, out_dtype);
}

}  // namespace pkv
