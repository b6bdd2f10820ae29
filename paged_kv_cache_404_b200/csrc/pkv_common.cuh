// pkv_common.cuh -- shared device helpers and the decode workspace layout.
//
// Everything here is written for sm_100a (B200).  The PTX wrappers cover the
// asynchronous copy engine (TMA tensor loads completing on an mbarrier), the
// warp-level tensor-core instruction used for the grouped-query contraction,
// and matrix fragment loads/transposes out of shared memory.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace pkv {

constexpr int kBlockSize = 16;

// ------------------------------------------------------------------ workspace
//
// Decode workspace (caller-allocated device memory), in this order:
//   WsHeader                       256 bytes
//   nparts   int32 [num_seqs]      partitions of each sequence (written by the plan)
//   items    int4  [num_seqs * max_parts]   (seq, partition, first block, blocks) work list
//   part_ml  float2[num_seqs * num_heads * max_parts]   (m, l) per partition
//   part_o   float [num_seqs * num_heads * max_parts * head_dim]
// and, for the shared-prefix decode only (written by the plan):
//   seq_sub     int32 [num_seqs]   subgroup of each sequence, -1 = none
//   seq_k       int32 [num_seqs]   leading blocks the sequence shares with its subgroup
//   sub_info    int4  [num_seqs]   (first member, members, shared blocks, 0) per subgroup
//   sub_members int32 [num_seqs]   member sequences, subgroup by subgroup
// Each region starts on a 256-byte boundary.
struct WsHeader {
    int counter;        // next unit to hand out (zeroed by the plan kernel)
    int num_items;      // (seq, partition, block range) items in the work list
    int num_units;      // num_items * num_kv_heads
    int partition;      // largest partition in tokens chosen for this call
    int timeout;        // set when a bounded wait ran out
    int num_subs;       // shared-prefix subgroups built by the plan
    int num_members;    // sequences in those subgroups
    int pad[57];
};
static_assert(sizeof(WsHeader) == 256, "header is one 256-byte line");

struct WsLayout {
    size_t nparts, items, part_ml, part_o, seq_sub, seq_k, sub_info, sub_members, total;
    int max_parts;
};

__host__ __device__ inline size_t pkv_align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline WsLayout ws_layout(int num_seqs, int num_heads, int head_dim, int max_parts) {
    WsLayout L;
    size_t off = sizeof(WsHeader);
    L.max_parts = max_parts;
    L.nparts = off;
    off = pkv_align256(off + sizeof(int) * (size_t)num_seqs);
    L.items = off;
    off = pkv_align256(off + sizeof(int4) * (size_t)num_seqs * max_parts);
    L.part_ml = off;
    off = pkv_align256(off + sizeof(float2) * (size_t)num_seqs * num_heads * max_parts);
    L.part_o = off;
    off = pkv_align256(off + sizeof(float) * (size_t)num_seqs * num_heads * max_parts * head_dim);
    L.seq_sub = L.seq_k = L.sub_info = L.sub_members = 0;
    L.total = off;
    return L;
}

// Layout of the shared-prefix decode: one more partition per sequence (its
// shared and its own blocks are cut separately) and the subgroup arrays.
__host__ __device__ inline WsLayout ws_layout_shared(int num_seqs, int num_heads, int head_dim, int max_parts) {
    WsLayout L = ws_layout(num_seqs, num_heads, head_dim, max_parts + 1);
    size_t off = L.total;
    L.seq_sub = off;
    off = pkv_align256(off + sizeof(int) * (size_t)num_seqs);
    L.seq_k = off;
    off = pkv_align256(off + sizeof(int) * (size_t)num_seqs);
    L.sub_info = off;
    off = pkv_align256(off + sizeof(int4) * (size_t)num_seqs);
    L.sub_members = off;
    off = pkv_align256(off + sizeof(int) * (size_t)num_seqs);
    L.total = off;
    return L;
}

// Everything the decode kernels need besides the tensor maps.
struct DecodeParams {
    void* out;
    const void* q;
    const int32_t* block_tables;
    const int32_t* context_lens;
    int max_blocks_per_seq;
    int num_seqs;
    int max_context_len;
    int num_blocks;
    int num_heads;
    int num_kv_heads;
    int group;
    int head_dim;
    float score_scale;   // scale * log2(e) (* k_scale for FP8): scores in base-2 units
    float out_scale;     // v_scale for FP8, else 1
    const void* k_pool;  // plain pointers (the CUDA-core path reads them directly)
    const void* v_pool;
    WsHeader* hdr;
    int* nparts;         // written by the plan kernel
    int4* items;         // written by the plan kernel: {seq, partition, first block, blocks}
    float2* part_ml;
    float* part_o;
    int max_parts;
    int32_t* err;
    // Shared-prefix groups (num_groups == 0: none).  Hints from the caller:
    // group g lists sequences group_seqs[group_offsets[g] .. group_offsets[g+1])
    // that claim to share their first group_shared_blocks[g] blocks.
    const int32_t* group_offsets;
    const int32_t* group_seqs;
    const int32_t* group_shared_blocks;
    int num_groups;
    int num_group_seqs;  // entries of group_seqs (offsets are clamped to it)
    int group_cap;       // members per subgroup: their query heads fill 16 score columns
    int* seq_sub;        // the plan's checked subgroups (workspace)
    int* seq_k;
    int4* sub_info;
    int* sub_members;
};

// Everything the prefill kernel needs besides the tensor maps.
struct PrefillParams {
    __nv_bfloat16* out;
    const __nv_bfloat16* q;
    const int32_t* block_tables;
    const int32_t* context_lens;
    const int32_t* query_start;
    int max_blocks_per_seq;
    int num_seqs;
    int num_blocks;
    int num_heads;
    int group;
    float score_scale;  // scale * k_scale * log2(e)
    float out_scale;    // v_scale (1 for a bf16 cache)
    int32_t* err;
};

// ------------------------------------------------------------------ small helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void count_error(int32_t* err, int n = 1) {
    if (err != nullptr) atomicAdd(err, n);
}

// Context length of sequence s clamped to what the table and the workspace can
// hold; a clamp is a device-data error.
__device__ __forceinline__ int clamped_len(const DecodeParams& p, int s, bool count) {
    int L = p.context_lens[s];
    int cap = p.max_blocks_per_seq * kBlockSize;
    if (p.max_context_len < cap) cap = p.max_context_len;
    if (L < 0 || L > cap) {
        if (count) count_error(p.err);
        L = L < 0 ? 0 : cap;
    }
    return L;
}

// Launch with programmatic stream serialisation (the kernel calls pdl_wait()
// before it touches memory the previous kernel on the stream may use).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for phase `parity` of an mbarrier: gives up after roughly
// `limit_cycles` SM clock cycles and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  long long limit_cycles = (1LL << 32)) {
    if (mbar_try_wait(bar, parity)) return true;
    long long t0 = clock64();
    for (;;) {
        #pragma unroll 1
        for (int i = 0; i < 256; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > limit_cycles) return false;
    }
}

// ------------------------------------------------------------------ launch ordering

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while the previous kernel on the stream finishes;
// pdl_wait() blocks until that kernel has completed and its memory is visible.
// Every kernel here calls pdl_wait() before touching memory another kernel may
// use, and pdl_trigger() once the next kernel may begin its own prologue.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ TMA

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled tensor load into shared memory, completing on mbarrier `bar`.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

// ------------------------------------------------------------------ fragments / MMA

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                            uint32_t& r3) {
    asm("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3) {
    asm("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

// D(16x8, f32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D(16x8, f32) += A(16x16, f16, row) * B(16x8, f16, col)
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two E4M3 codes (low byte -> low half) to two f16 values; exact (every E4M3
// value is representable in f16).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes & 0xFFFFu), __NV_E4M3);
    return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace pkv
