// api.cu -- the C ABI declared in include/pagedkv.h: argument validation,
// TMA descriptor encoding and kernel launches.  No memory is allocated here;
// every buffer belongs to the caller.
#include <cudaTypedefs.h>

#include <cmath>

#include "pagedkv.h"
#include "pkv_common.cuh"

namespace pkv {
cudaError_t launch_kv_write(const void* k, const void* v, int src_dtype, const int64_t* slots, int num_tokens,
                            void* k_pool, void* v_pool, int cache_dtype, long long num_slots, int row_elems,
                            float k_scale, float v_scale, int32_t* err, cudaStream_t stream);
cudaError_t launch_copy_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v, size_t block_bytes,
                               const int64_t* pairs, int num_pairs, int src_blocks, int dst_blocks, int32_t* err,
                               cudaStream_t stream);
cudaError_t launch_decode_plan(const DecodeParams& p, int fixed_partition, int min_partition, int num_candidates,
                               int target_units, int out_dtype, cudaStream_t stream);
cudaError_t launch_decode_tc(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecodeParams& p, bool fp8,
                             int num_sms, cudaStream_t stream);
cudaError_t launch_decode_f32(const DecodeParams& p, int num_sms, cudaStream_t stream);
int decode_tc_warps(bool fp8, int head_dim, bool grouped);
bool decode_tc_groupable(bool fp8, int head_dim, int group);
cudaError_t launch_decode_merge(const DecodeParams& p, int out_dtype, int num_sms, cudaStream_t stream);
cudaError_t launch_prefill_tc(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                              const PrefillParams& p, bool fp8, int max_query_len, cudaStream_t stream);
}  // namespace pkv

using namespace pkv;

namespace {

// Smallest partition the automatic plan considers for a batch whose workspace
// is large (see min_partition_of), and how many units per warp it aims for
// before it stops halving the partition.
constexpr int kMinAutoPartition = 256;
constexpr int kUnitsPerWorker = 3;
constexpr int kMaxCandidates = 12;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t elem_bytes(int dt) { return dt == PKV_F32 ? 4 : dt == PKV_BF16 ? 2 : 1; }

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    return n;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// Tensor map over a pool viewed as [slots][kv heads][head_dim]; box = 16 slots
// x 1 head x 128 bytes, 128-byte swizzle (conflict-free ldmatrix of 16 rows).
bool pool_tensor_map(CUtensorMap* map, const void* pool, int cache_dtype, int head_dim, int num_kv_heads,
                     long long num_slots) {
    auto enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t es = elem_bytes(cache_dtype);
    const cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_kv_heads, (cuuint64_t)num_slots};
    const cuuint64_t strides[2] = {(cuuint64_t)head_dim * es, (cuuint64_t)head_dim * num_kv_heads * es};
    const cuuint32_t box[3] = {(cuuint32_t)(128 / es), 1, (cuuint32_t)kBlockSize};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType dt =
        cache_dtype == PKV_FP8_E4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUresult r = enc(map, dt, 3, const_cast<void*>(pool), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// bf16 tensor [rows][heads][head_dim]: box of box_rows rows x 1 head x 128 bytes,
// 128-byte swizzle; rows past the end read zeros.
bool rows_tensor_map(CUtensorMap* map, const void* base, int head_dim, int heads, long long rows, int box_rows) {
    auto enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)heads, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, (cuuint64_t)head_dim * heads * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Workspace within which automatic partitioning may cut below kMinAutoPartition
// tokens (at most the no-alloc decode's scratch, so that whatever that entry point
// accepted with 256-token pieces it still accepts), and the smaller partition.
constexpr size_t kSmallBatchWorkspace = PKV_NOALLOC_SCRATCH_BYTES;
constexpr int kSmallBatchPartition = 128;

int parts_for(int max_context_len, int P) {
    const int n = (max_context_len + P - 1) / P;
    return n > 0 ? n : 1;
}

// Smallest partition the plan may use.  A fixed partition is the caller's.
// Automatic: 256 tokens, or 128 when the workspace for 128-token pieces stays
// within kSmallBatchWorkspace -- a small batch then gets enough pieces to keep
// the warps busy (few sequences would otherwise leave most warps idle while each
// walks a long piece); large batches have the work already.  (64-token pieces
// were measured too: the beam step's decode call took 61 us against 51 with
// 128, the extra partitions costing the plan and the merge more than they gave.)
int min_partition_of(int partition_tokens, int num_seqs, int num_heads, int head_dim, int max_context_len,
                     bool shared) {
    if (partition_tokens > 0) return partition_tokens;
    const int parts = parts_for(max_context_len, kSmallBatchPartition);
    const size_t bytes = shared ? ws_layout_shared(num_seqs, num_heads, head_dim, parts).total
                                : ws_layout(num_seqs, num_heads, head_dim, parts).total;
    return bytes <= kSmallBatchWorkspace ? kSmallBatchPartition : kMinAutoPartition;
}

int max_parts_of(int partition_tokens, int num_seqs, int num_heads, int head_dim, int max_context_len, bool shared) {
    return parts_for(max_context_len,
                     min_partition_of(partition_tokens, num_seqs, num_heads, head_dim, max_context_len, shared));
}

// Optional shared-prefix hints of pkv_paged_attention_decode_shared.
struct PrefixGroups {
    const int32_t* offsets = nullptr;
    const int32_t* seqs = nullptr;
    const int32_t* shared_blocks = nullptr;
    int num_seqs = 0;
    int num_groups = 0;
    bool layout = false;  // workspace laid out by ws_layout_shared
};

int decode_impl(void* out, const void* q, int q_dtype, const void* k_pool, const void* v_pool, int cache_dtype,
                const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                int max_context_len, int num_blocks, int block_size, int num_heads, int num_kv_heads, int head_dim,
                float scale, float k_scale, float v_scale, int partition_tokens, const PrefixGroups& pg,
                void* workspace, size_t workspace_bytes, int32_t* err_count, void* stream);

}  // namespace

extern "C" {

const char* pkv_status_string(int status) {
    switch (status) {
        case PKV_OK: return "ok";
        case PKV_EINVAL: return "invalid argument";
        case PKV_EUNSUPPORTED: return "unsupported configuration";
        case PKV_ECUDA: return "CUDA error";
        case PKV_ENOMEM: return "out of free blocks";
        case PKV_ENOENT: return "no such sequence";
        case PKV_ESWAPPED: return "sequence is swapped out to the host pool";
        default: return "unknown status";
    }
}

int pkv_version(void) { return PKV_VERSION; }

int pkv_paged_kv_write(const void* k, const void* v, int src_dtype, const int64_t* slot_mapping, int num_tokens,
                       void* k_pool, void* v_pool, int cache_dtype, int num_blocks, int block_size,
                       int num_kv_heads, int head_dim, float k_scale, float v_scale, int32_t* err_count,
                       void* stream) {
    if (num_tokens < 0 || num_blocks <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0)
        return PKV_EINVAL;
    if (block_size != kBlockSize) return PKV_EUNSUPPORTED;
    const bool same = src_dtype == cache_dtype && (src_dtype == PKV_F32 || src_dtype == PKV_BF16);
    const bool quant = cache_dtype == PKV_FP8_E4M3 && (src_dtype == PKV_BF16 || src_dtype == PKV_F32);
    if (!same && !quant) return PKV_EUNSUPPORTED;
    const long long row = (long long)num_kv_heads * head_dim;
    if (same && (row * (long long)elem_bytes(src_dtype)) % 16 != 0) return PKV_EUNSUPPORTED;
    if (quant && row % 16 != 0) return PKV_EUNSUPPORTED;
    if (cache_dtype == PKV_FP8_E4M3 && !(k_scale > 0.f && v_scale > 0.f)) return PKV_EINVAL;
    if (num_tokens == 0) return PKV_OK;
    if (!k || !v || !slot_mapping || !k_pool || !v_pool) return PKV_EINVAL;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) ||
        !aligned(slot_mapping, 8) || !aligned(err_count, 4))
        return PKV_EINVAL;
    cudaError_t e = launch_kv_write(k, v, src_dtype, slot_mapping, num_tokens, k_pool, v_pool, cache_dtype,
                                    (long long)num_blocks * block_size, (int)row, k_scale, v_scale, err_count,
                                    static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

size_t pkv_decode_workspace_bytes(int num_seqs, int num_heads, int head_dim, int max_context_len,
                                  int partition_tokens) {
    if (num_seqs < 0 || num_heads <= 0 || head_dim <= 0 || max_context_len < 0 || partition_tokens < 0 ||
        partition_tokens % kBlockSize != 0)
        return 0;
    return ws_layout(num_seqs, num_heads, head_dim,
                     max_parts_of(partition_tokens, num_seqs, num_heads, head_dim, max_context_len, false))
        .total;
}

int pkv_paged_attention_decode(void* out, const void* q, int q_dtype, const void* k_pool, const void* v_pool,
                               int cache_dtype, const int32_t* block_tables, int max_blocks_per_seq,
                               const int32_t* context_lens, int num_seqs, int max_context_len, int num_blocks,
                               int block_size, int num_heads, int num_kv_heads, int head_dim, float scale,
                               float k_scale, float v_scale, int partition_tokens, void* workspace,
                               size_t workspace_bytes, int32_t* err_count, void* stream) {
    return decode_impl(out, q, q_dtype, k_pool, v_pool, cache_dtype, block_tables, max_blocks_per_seq, context_lens,
                       num_seqs, max_context_len, num_blocks, block_size, num_heads, num_kv_heads, head_dim, scale,
                       k_scale, v_scale, partition_tokens, PrefixGroups(), workspace, workspace_bytes, err_count,
                       stream);
}

size_t pkv_decode_workspace_bytes_shared(int num_seqs, int num_heads, int head_dim, int max_context_len,
                                         int partition_tokens) {
    if (num_seqs < 0 || num_heads <= 0 || head_dim <= 0 || max_context_len < 0 || partition_tokens < 0 ||
        partition_tokens % kBlockSize != 0)
        return 0;
    return ws_layout_shared(num_seqs, num_heads, head_dim,
                            max_parts_of(partition_tokens, num_seqs, num_heads, head_dim, max_context_len, true))
        .total;
}

int pkv_paged_attention_decode_shared(void* out, const void* q, int q_dtype, const void* k_pool, const void* v_pool,
                                      int cache_dtype, const int32_t* block_tables, int max_blocks_per_seq,
                                      const int32_t* context_lens, int num_seqs, int max_context_len,
                                      int num_blocks, int block_size, int num_heads, int num_kv_heads, int head_dim,
                                      float scale, float k_scale, float v_scale, int partition_tokens,
                                      const int32_t* group_offsets, const int32_t* group_seqs, int num_group_seqs,
                                      const int32_t* group_shared_blocks, int num_groups, void* workspace,
                                      size_t workspace_bytes, int32_t* err_count, void* stream) {
    if (num_groups < 0 || num_group_seqs < 0) return PKV_EINVAL;
    PrefixGroups pg;
    pg.layout = true;
    if (num_groups > 0 && num_group_seqs > 0) {
        if (!group_offsets || !group_seqs || !group_shared_blocks) return PKV_EINVAL;
        if (!aligned(group_offsets, 4) || !aligned(group_seqs, 4) || !aligned(group_shared_blocks, 4))
            return PKV_EINVAL;
        pg.offsets = group_offsets;
        pg.seqs = group_seqs;
        pg.shared_blocks = group_shared_blocks;
        pg.num_seqs = num_group_seqs;
        pg.num_groups = num_groups;
    }
    return decode_impl(out, q, q_dtype, k_pool, v_pool, cache_dtype, block_tables, max_blocks_per_seq, context_lens,
                       num_seqs, max_context_len, num_blocks, block_size, num_heads, num_kv_heads, head_dim, scale,
                       k_scale, v_scale, partition_tokens, pg, workspace, workspace_bytes, err_count, stream);
}

}  // extern "C"

namespace pkv {

// Every host-side check of the decode except those of its workspace; PKV_OK
// with num_seqs == 0 means there is nothing to launch.
int decode_check_args(const void* out, const void* q, int q_dtype, const void* k_pool, const void* v_pool,
                      int cache_dtype, const int32_t* block_tables, int max_blocks_per_seq,
                      const int32_t* context_lens, int num_seqs, int max_context_len, int num_blocks, int block_size,
                      int num_heads, int num_kv_heads, int head_dim, float k_scale, float v_scale,
                      int partition_tokens, const int32_t* err_count) {
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || max_context_len < 0 || num_blocks <= 0 || block_size <= 0 ||
        num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || partition_tokens < 0)
        return PKV_EINVAL;
    if (num_heads % num_kv_heads != 0) return PKV_EINVAL;
    if (partition_tokens % kBlockSize != 0) return PKV_EINVAL;
    if (block_size != kBlockSize) return PKV_EUNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return PKV_EUNSUPPORTED;
    const bool f32 = q_dtype == PKV_F32 && cache_dtype == PKV_F32;
    const bool bf16 = q_dtype == PKV_BF16 && cache_dtype == PKV_BF16;
    const bool fp8 = q_dtype == PKV_BF16 && cache_dtype == PKV_FP8_E4M3;
    if (!f32 && !bf16 && !fp8) return PKV_EUNSUPPORTED;
    if (!f32 && num_heads / num_kv_heads > 16) return PKV_EUNSUPPORTED;
    if (fp8 && head_dim != 128) return PKV_EUNSUPPORTED;
    if (fp8 && !(k_scale > 0.f && v_scale > 0.f)) return PKV_EINVAL;
    if (num_seqs == 0) return PKV_OK;
    if (!out || !q || !k_pool || !v_pool || !block_tables || !context_lens) return PKV_EINVAL;
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(err_count, 4))
        return PKV_EINVAL;
    return PKV_OK;
}

}  // namespace pkv

namespace {

int decode_impl(void* out, const void* q, int q_dtype, const void* k_pool, const void* v_pool, int cache_dtype,
                const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                int max_context_len, int num_blocks, int block_size, int num_heads, int num_kv_heads, int head_dim,
                float scale, float k_scale, float v_scale, int partition_tokens, const PrefixGroups& pg,
                void* workspace, size_t workspace_bytes, int32_t* err_count, void* stream) {
    const int status = decode_check_args(out, q, q_dtype, k_pool, v_pool, cache_dtype, block_tables,
                                         max_blocks_per_seq, context_lens, num_seqs, max_context_len, num_blocks,
                                         block_size, num_heads, num_kv_heads, head_dim, k_scale, v_scale,
                                         partition_tokens, err_count);
    if (status != PKV_OK || num_seqs == 0) return status;
    if (!workspace || !aligned(workspace, 256)) return PKV_EINVAL;
    const bool f32 = q_dtype == PKV_F32;
    const bool fp8 = cache_dtype == PKV_FP8_E4M3;
    const int group = num_heads / num_kv_heads;
    const int max_parts =
        max_parts_of(partition_tokens, num_seqs, num_heads, head_dim, max_context_len, pg.layout);
    const WsLayout ws = pg.layout ? ws_layout_shared(num_seqs, num_heads, head_dim, max_parts)
                                  : ws_layout(num_seqs, num_heads, head_dim, max_parts);
    if (workspace_bytes < ws.total) return PKV_EINVAL;
    // groups only where a grouped kernel exists and two members fit in 16 columns
    const bool grouped = pg.num_groups > 0 && !f32 && decode_tc_groupable(fp8, head_dim, group);

    const int num_sms = sm_count();
    if (num_sms <= 0) return PKV_ECUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    char* w = static_cast<char*>(workspace);
    DecodeParams p;
    p.out = out;
    p.q = q;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_seqs = num_seqs;
    p.max_context_len = max_context_len;
    p.num_blocks = num_blocks;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.group = group;
    p.head_dim = head_dim;
    const float log2e = 1.4426950408889634f;
    p.score_scale = scale * log2e * (fp8 ? k_scale : 1.f);
    p.out_scale = fp8 ? v_scale : 1.f;
    p.k_pool = k_pool;
    p.v_pool = v_pool;
    p.hdr = reinterpret_cast<WsHeader*>(w);
    p.nparts = reinterpret_cast<int*>(w + ws.nparts);
    p.items = reinterpret_cast<int4*>(w + ws.items);
    p.part_ml = reinterpret_cast<float2*>(w + ws.part_ml);
    p.part_o = reinterpret_cast<float*>(w + ws.part_o);
    p.max_parts = ws.max_parts;
    p.err = err_count;
    p.group_offsets = grouped ? pg.offsets : nullptr;
    p.group_seqs = grouped ? pg.seqs : nullptr;
    p.group_shared_blocks = grouped ? pg.shared_blocks : nullptr;
    p.num_groups = grouped ? pg.num_groups : 0;
    p.num_group_seqs = grouped ? pg.num_seqs : 0;
    p.group_cap = 16 / group;
    p.seq_sub = pg.layout ? reinterpret_cast<int*>(w + ws.seq_sub) : nullptr;
    p.seq_k = pg.layout ? reinterpret_cast<int*>(w + ws.seq_k) : nullptr;
    p.sub_info = pg.layout ? reinterpret_cast<int4*>(w + ws.sub_info) : nullptr;
    p.sub_members = pg.layout ? reinterpret_cast<int*>(w + ws.sub_members) : nullptr;

    // Partition candidates: min_partition << c, up to the first that covers max_context_len.
    const int min_p = min_partition_of(partition_tokens, num_seqs, num_heads, head_dim, max_context_len, pg.layout);
    int ncand = 1;
    if (partition_tokens == 0)
        while (ncand < kMaxCandidates && ((long long)min_p << (ncand - 1)) < max_context_len) ++ncand;
    const int warps_per_sm = f32 ? 32 : decode_tc_warps(fp8, head_dim, grouped);
    const int target_units = num_sms * warps_per_sm * kUnitsPerWorker;
    const int out_dtype = f32 ? 0 : 1;

    cudaError_t e = launch_decode_plan(p, partition_tokens, min_p, ncand, target_units, out_dtype, st);
    if (e != cudaSuccess) return PKV_ECUDA;
    if (f32) {
        e = launch_decode_f32(p, num_sms, st);
    } else {
        CUtensorMap tmK, tmV;
        const long long slots = (long long)num_blocks * block_size;
        if (!pool_tensor_map(&tmK, k_pool, cache_dtype, head_dim, num_kv_heads, slots) ||
            !pool_tensor_map(&tmV, v_pool, cache_dtype, head_dim, num_kv_heads, slots))
            return PKV_ECUDA;
        e = launch_decode_tc(tmK, tmV, p, fp8, num_sms, st);
    }
    if (e != cudaSuccess) return PKV_ECUDA;
    // a split (and so a merge) is possible only if the smallest partition is
    // shorter than the longest context, or if a sequence's shared and own
    // blocks are cut apart
    if (grouped || min_p < max_context_len) {
        e = launch_decode_merge(p, out_dtype, num_sms, st);
        if (e != cudaSuccess) return PKV_ECUDA;
    }
    return PKV_OK;
}

}  // namespace

extern "C" {

int pkv_paged_attention_prefill(void* out, const void* q, int q_dtype, const void* k_pool, const void* v_pool,
                                int cache_dtype, const int32_t* block_tables, int max_blocks_per_seq,
                                const int32_t* context_lens, const int32_t* query_start, int num_seqs,
                                int total_query_tokens, int max_query_len, int num_blocks, int block_size,
                                int num_heads, int num_kv_heads, int head_dim, float scale, float k_scale,
                                float v_scale, int32_t* err_count, void* stream) {
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || max_query_len < 0 || total_query_tokens < 0 || num_blocks <= 0 ||
        block_size <= 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0)
        return PKV_EINVAL;
    if (num_heads % num_kv_heads != 0) return PKV_EINVAL;
    if (block_size != kBlockSize) return PKV_EUNSUPPORTED;
    const bool fp8 = cache_dtype == PKV_FP8_E4M3;
    if (q_dtype != PKV_BF16 || (cache_dtype != PKV_BF16 && !fp8) || head_dim != 128) return PKV_EUNSUPPORTED;
    if (fp8 && !(std::isfinite(k_scale) && std::isfinite(v_scale))) return PKV_EINVAL;
    if (num_seqs == 0 || max_query_len == 0 || total_query_tokens == 0) return PKV_OK;
    // grid (heads, 256-row query tiles, sequences): y and z are limited to 65535
    if (num_seqs > 65535 || num_heads > 65535 || (max_query_len + 255) / 256 > 65535) return PKV_EUNSUPPORTED;
    if (!out || !q || !k_pool || !v_pool || !block_tables || !context_lens || !query_start) return PKV_EINVAL;
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(query_start, 4) || !aligned(err_count, 4))
        return PKV_EINVAL;
    PrefillParams p;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.query_start = query_start;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_seqs = num_seqs;
    p.num_blocks = num_blocks;
    p.num_heads = num_heads;
    p.group = num_heads / num_kv_heads;
    p.score_scale = scale * (fp8 ? k_scale : 1.f) * 1.4426950408889634f;
    p.out_scale = fp8 ? v_scale : 1.f;
    p.err = err_count;
    CUtensorMap tmK, tmV;
    const long long slots = (long long)num_blocks * block_size;
    if (!pool_tensor_map(&tmK, k_pool, cache_dtype, head_dim, num_kv_heads, slots) ||
        !pool_tensor_map(&tmV, v_pool, cache_dtype, head_dim, num_kv_heads, slots))
        return PKV_ECUDA;
    // q viewed as [total_q][heads][head_dim]; boxes of 128 rows x 1 head x 128 bytes
    CUtensorMap tmQ;
    if (!rows_tensor_map(&tmQ, q, head_dim, num_heads, total_query_tokens, 128)) return PKV_ECUDA;
    const cudaError_t e = launch_prefill_tc(tmQ, tmK, tmV, p, fp8, max_query_len, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

int pkv_copy_blocks(void* k_pool, void* v_pool, size_t block_bytes, const int64_t* src_dst_pairs, int num_pairs,
                    int num_blocks, int32_t* err_count, void* stream) {
    if (num_pairs < 0 || num_blocks <= 0 || block_bytes == 0 || block_bytes % 16 != 0) return PKV_EINVAL;
    if (num_pairs == 0) return PKV_OK;
    if (!k_pool || !v_pool || !src_dst_pairs) return PKV_EINVAL;
    if (!aligned(k_pool, 16) || !aligned(v_pool, 16) || !aligned(src_dst_pairs, 8) || !aligned(err_count, 4))
        return PKV_EINVAL;
    // grid.y carries the pair index: launch in slices of at most 65535 pairs
    for (int first = 0; first < num_pairs; first += 65535) {
        const int n = num_pairs - first < 65535 ? num_pairs - first : 65535;
        cudaError_t e = launch_copy_blocks(k_pool, v_pool, k_pool, v_pool, block_bytes,
                                           src_dst_pairs + 2 * (size_t)first, n, num_blocks, num_blocks, err_count,
                                           static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return PKV_ECUDA;
    }
    return PKV_OK;
}

}  // extern "C"

namespace {

// Address the device uses for `p`: device or managed memory as is, page-locked
// host memory through its device mapping; nullptr if the device cannot reach it
// (pageable host memory, unknown pointer).
const void* device_view(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();  // clear the error this query left as the runtime's last error
        return nullptr;
    }
    if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return p;
    if (a.type == cudaMemoryTypeHost) return a.devicePointer;
    return nullptr;
}

}  // namespace

extern "C" {

int pkv_swap_blocks(void* dst_k_pool, void* dst_v_pool, int dst_num_blocks, const void* src_k_pool,
                    const void* src_v_pool, int src_num_blocks, size_t block_bytes, const int64_t* src_dst_pairs,
                    int num_pairs, int32_t* err_count, void* stream) {
    if (num_pairs < 0 || dst_num_blocks <= 0 || src_num_blocks <= 0 || block_bytes == 0 || block_bytes % 16 != 0)
        return PKV_EINVAL;
    if (num_pairs == 0) return PKV_OK;
    if (!dst_k_pool || !dst_v_pool || !src_k_pool || !src_v_pool || !src_dst_pairs) return PKV_EINVAL;
    if (!aligned(dst_k_pool, 16) || !aligned(dst_v_pool, 16) || !aligned(src_k_pool, 16) ||
        !aligned(src_v_pool, 16) || !aligned(src_dst_pairs, 8) || !aligned(err_count, 4))
        return PKV_EINVAL;
    void* dk = const_cast<void*>(device_view(dst_k_pool));
    void* dv = const_cast<void*>(device_view(dst_v_pool));
    const void* sk = device_view(src_k_pool);
    const void* sv = device_view(src_v_pool);
    const int64_t* pr = static_cast<const int64_t*>(device_view(src_dst_pairs));
    if (!dk || !dv || !sk || !sv || !pr) return PKV_EINVAL;
    for (int first = 0; first < num_pairs; first += 65535) {
        const int n = num_pairs - first < 65535 ? num_pairs - first : 65535;
        cudaError_t e = launch_copy_blocks(dk, dv, sk, sv, block_bytes, pr + 2 * (size_t)first, n, src_num_blocks,
                                           dst_num_blocks, err_count, static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return PKV_ECUDA;
    }
    return PKV_OK;
}

}  // extern "C"
