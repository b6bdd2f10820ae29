// prefill_tc.cu -- causal multi-token paged attention (the prompt pass) on the
// 5th-generation tensor cores (tcgen05).
//
// What it computes: sequence s has nq new query tokens, the last nq of its
// context_len tokens (K/V already in the pool); query i at position
// p = context_len - nq + i attends to every token t <= p through the block table
// (iplexlaw.co.kr, logical vs physical order; gyaansetu.com, what the KV cache
// holds).
//
// Two kernels, one per cache type; both take one CTA per (sequence, 256 query rows
// = two Q tiles of 128, query head), on a grid ordered (head, tile, sequence) so that
// a sequence's CTAs run together and its last rows come first, hold O and the scores
// of both Q tiles in the
// 512 TMEM columns, and split the work between warps: a producer (TMA loads of Q
// once and of K/V tiles through the block table, with the V rows that hold no token
// zeroed in shared memory, so that a zero probability never meets a NaN there), an
// MMA issuer (runs warp-uniformly, one elected lane issuing tcgen05.mma; commits
// signal mbarriers) and two softmax warpgroups, one per Q tile, in which thread r
// owns query row r (TMEM lane r): it loads the row's scores with tcgen05.ld, masks
// the causal boundary and the blocks with no token, runs the online softmax in base
// 2 (the reference max moves only when a score exceeds it by more than 2^8, then O
// is rescaled in TMEM), writes P as 16-bit pairs into TMEM over the scores it has
// read, and finally normalises O and stores the row.  The tensor core runs one
// thread's products in issue order, so a score product issued after PV_t(j) may
// overwrite the P it reads, and the commit that follows it also covers PV_t(j).
//
// bf16 cache (prefill_bf16_kernel, twelve warps): 128-key tiles, so that the score
// products are M = N = 128, K = 128 (full tensor-core rate; N = 64 products need
// their operands from shared memory faster than it delivers them), K and V in 2-stage
// rings apart (192 KB with the Q tiles; 3 stages of either measured slower), one score
// buffer per Q tile.
// Per KV tile j the issuer runs PV_0(j), S_0(j+1), PV_1(j), S_1(j+1): while one Q
// tile's softmax runs, the tensor core does the other Q tile's products.
//
// FP8 E4M3 cache (prefill_fp8_kernel, 14 warps): 64-key tiles with two score buffers
// per Q tile, K/V in a 4-stage ring of f16 tiles.  The products run in f16, which
// holds every E4M3 value exactly.  Warp 8 TMA-loads the codes (128-byte rows) into a
// 2-deep staging ring; warps 10-13 each turn one 16-slot block of a tile into f16
// in the ring the tensor core reads (and zero V where no token is), then arrive on
// the stage's barriers; the softmax warps first turn their Q tile from bf16 into
// f16 in place and write P as f16.  k_scale folds into the score scale and v_scale
// into the final normalisation.  S_t(j+2) is issued right after PV_t(j), so the
// softmax of tile j+1 runs while the tensor core does PV_t(j) and S_t(j+2).
#include "pkv_common.cuh"

namespace pkv {

namespace {

constexpr int kTcRows = 128;                   // query rows per Q tile (MMA M)
constexpr int kTcQT = 2;                       // Q tiles per CTA (two softmax warpgroups, ping-pong)
constexpr int kTcKeys = 64;                    // FP8 kernel: keys per KV tile (MMA N of S, K of PV)
constexpr int kTcD = 128;                      // head_dim
constexpr int kTcQChunk = kTcRows * 128;       // one 64-element column chunk of a 128-row operand: 16 KB
constexpr int kTcQBytes = 2 * kTcQChunk;       // Q tile: 128 rows x 128 bf16
constexpr int kTcKVChunk = kTcKeys * 128;      // one 64-element column chunk of a 64-row operand: 8 KB
constexpr int kTcKVBytes = 2 * kTcKVChunk;     // K (or V) tile: 64 keys x 128 bf16
constexpr int kTcStages = 4;
constexpr int kTcBlocks = kTcKeys / kBlockSize;  // table blocks per KV tile
// shared memory layout (offsets from a 1024-aligned base)
constexpr int kTcQ = 0;                                    // Q tile t at kTcQ + t * kTcQBytes (TMA landing)
constexpr int kTcKV = kTcQ + kTcQT * kTcQBytes;            // stage st: K, then V
constexpr int kTcSmem = kTcKV + kTcStages * 2 * kTcKVBytes;  // 192 KB
// FP8 cache: E4M3 K and V tiles land in a 2-deep staging ring (64 rows x 128 bytes
// each), then become f16 in the ring above
constexpr int kTcStgBytes = kTcKeys * 128;
constexpr int kTcStg = kTcSmem;
constexpr int kTcSmemFp8 = kTcStg + 2 * 2 * kTcStgBytes;  // 224 KB
// TMEM columns (512): O of Q tile t at t*128 (fp32); scores of Q tile t, KV tile j in
// buffer 256 + (2t + (j & 1))*64 (fp32; P as 16-bit pairs over its first 32)
constexpr int kTcOCol = 0, kTcSCol = 256;
constexpr float kRescaleThreshold = 8.f;       // log2 of the largest factor p may exceed 1 by
constexpr int kTcOkWords = 64;                 // validity bits kept in shared memory for 2048 blocks

// ---- tcgen05 wrappers -----------------------------------------------------------

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor, kind::f16: A and B both bf16 (or both f16), fp32 accumulator, M x N.
__host__ __device__ constexpr uint32_t instr_desc_16(int M, int N, bool b_mn_major, bool f16) {
    return (1u << 4) | ((f16 ? 0u : 1u) << 7) | ((f16 ? 0u : 1u) << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// 16 E4M3 codes (one 16-byte chunk) -> 16 f16 values in two 16-byte words (exact)
__device__ __forceinline__ void e4m3x16_to_f16(const uint4 c, uint4& lo, uint4& hi) {
    lo.x = e4m3x2_to_f16x2(c.x);
    lo.y = e4m3x2_to_f16x2(c.x >> 16);
    lo.z = e4m3x2_to_f16x2(c.y);
    lo.w = e4m3x2_to_f16x2(c.y >> 16);
    hi.x = e4m3x2_to_f16x2(c.z);
    hi.y = e4m3x2_to_f16x2(c.z >> 16);
    hi.z = e4m3x2_to_f16x2(c.w);
    hi.w = e4m3x2_to_f16x2(c.w >> 16);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// two bf16 (one word) times a power of two `up` -> two f16 (round to nearest)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t w, float up) {
    return pack_f16x2(__uint_as_float(w << 16) * up, __uint_as_float(w & 0xFFFF0000u) * up);
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive TMEM columns of this thread's lane (warp w reads lanes 32*(w%4)..).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }


// ---- 128-key tiles (bf16 cache) ------------------------------------------------
constexpr int kWKeys = 128;                        // keys per KV tile (MMA N of S, K of PV)
constexpr int kWChunk = kWKeys * 128;              // one 64-column chunk of a 128-row operand: 16 KB
constexpr int kWTile = 2 * kWChunk;                // K (or V) tile: 128 keys x 128 bf16
constexpr int kWKStages = 2, kWVStages = 2;        // K ring, V ring
constexpr int kWBlocks = kWKeys / kBlockSize;      // table blocks per KV tile
constexpr int kWK = kTcQT * kTcQBytes;             // shared memory: Q tiles, then the K ring, then the V ring
constexpr int kWV = kWK + kWKStages * kWTile;
constexpr int kWSmem = kWV + kWVStages * kWTile;   // 192 KB
constexpr int kWSCol = 256;                        // TMEM: O_t at 128 t, S_t at 256 + 128 t (P_t over its first 64)
static_assert(kWSmem + 1024 <= 227 * 1024, "shared memory");

// The issuing warp runs uniformly; elect.sync picks the one lane that issues, so
// every operand of the tensor-core instruction is warp-uniform.
__device__ __forceinline__ void umma_ss_e(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void umma_ts_e(uint32_t tmem_d, uint32_t tmem_a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void umma_commit_e(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
        : "memory");
}

// two fp32 in one 64-bit register pair, and the paired fp32 arithmetic
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// P of one row's 128 scores x (masked ones -inf): p = 2^(x * sc - mu) as bf16 pairs in
// pf, their sum returned; MASKED also zeroes the probabilities of masked scores (the
// argument of a masked score may be NaN when the scale is 0).
template <bool MASKED>
__device__ __forceinline__ float row_probs(const float (&x)[128], uint64_t sc2, uint64_t nmu2, int valid_to,
                                           unsigned okmask, uint32_t (&pf)[64]) {
    uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int e = 0; e < 64; ++e) {
        float a0, a1;
        f2_split(fma2(f2(x[2 * e], x[2 * e + 1]), sc2, nmu2), a0, a1);
        if (MASKED) {
            const bool blk = ((okmask >> ((2 * e) >> 4)) & 1u) != 0u;
            a0 = (2 * e <= valid_to && blk) ? a0 : -INFINITY;
            a1 = (2 * e + 1 <= valid_to && blk) ? a1 : -INFINITY;
        }
        const float p0 = fast_exp2(a0), p1 = fast_exp2(a1);
        sum2[e & 3] = add2(sum2[e & 3], f2(p0, p1));
        pf[e] = pack_bf16x2(p0, p1);
    }
    float s0, s1, s2, s3;
    f2_split(add2(sum2[0], sum2[1]), s0, s1);
    f2_split(add2(sum2[2], sum2[3]), s2, s3);
    return (s0 + s1) + (s2 + s3);
}

__device__ __forceinline__ void tmem_ld32_u(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

}  // namespace

__global__ void __launch_bounds__(448, 1)
    prefill_fp8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
    extern __shared__ uint8_t smem_raw[];
    // kv_full[S], kv_empty[S], v_ready[S] (S = kTcStages), q_full, s_full[2][2], p_full[2][2],
    // pv_done[2][2], stg_full[2], stg_empty[2], q_ready.  Scores, P and PV completion
    // have one barrier per (Q tile, buffer j & 1), so that no barrier is ever more than
    // one phase ahead of a waiter: the softmax may finish tile j+1 before the MMA issuer
    // takes P(j), and may skip PV waits while the reference max stays put.
    __shared__ __align__(8) uint64_t bars[3 * kTcStages + 18];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    __shared__ uint32_t ok_bits[kTcOkWords];  // block b of the sequence holds tokens (table, id in range)
    volatile int* abort_flag = &abort_sh;
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t b0 = smem_u32(&bars[0]);
    const uint32_t kv_full = b0, kv_empty = kv_full + 8 * kTcStages, v_ready = kv_empty + 8 * kTcStages,
                   q_full = v_ready + 8 * kTcStages, s_full = q_full + 8, p_full = s_full + 32, pv_done = p_full + 32,
                   stg_full = pv_done + 32, stg_empty = stg_full + 16, q_ready = stg_empty + 16;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kProducer = 8, kMma = 9, kConv0 = 10;  // warps 10-13 convert
    constexpr int kConvWarps = kTcBlocks;
    constexpr uint32_t kFull = 0xffffffffu;

    // grid (head, 256-row tile, sequence): a sequence's CTAs run together (its K/V
    // stays in L2 for all its tiles and heads), its last rows (the most KV tiles)
    // first, so that each sequence's CTAs reach the SMs longest first and end short
    const int h = blockIdx.x, s = blockIdx.z, kvh = h / p.group;
    const int tile = gridDim.y - 1 - blockIdx.y;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kTcStages; ++i) {
            mbar_init(kv_full + 8 * i, kConvWarps);
            mbar_init(kv_empty + 8 * i, 1);
            mbar_init(v_ready + 8 * i, kConvWarps);
        }
        mbar_init(q_full, 1);
        for (int i = 0; i < 2 * kTcQT; ++i) {
            mbar_init(s_full + 8 * i, 1);
            mbar_init(p_full + 8 * i, 4);
            mbar_init(pv_done + 8 * i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(stg_full + 8 * i, 1);
            mbar_init(stg_empty + 8 * i, kConvWarps);
        }
        mbar_init(q_ready, 8);  // each softmax warp has turned its share of Q into f16
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kProducer && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();

    const int qs0 = p.query_start[s];
    const int nq = p.query_start[s + 1] - qs0;
    const int ctx = p.context_lens[s];
    const int row0 = tile * (kTcQT * kTcRows);
    if (row0 >= nq) return;  // the whole CTA leaves together, before TMEM allocation
    if (nq > ctx || ctx > p.max_blocks_per_seq * kBlockSize) {
        if (tile == 0 && h == 0 && threadIdx.x == 0) count_error(p.err);
        const int rows = min(kTcQT * kTcRows, nq - row0);
        for (int e = threadIdx.x; e < rows * kTcD; e += blockDim.x) {
            const int r = e / kTcD, d = e - r * kTcD;
            p.out[((size_t)(qs0 + row0 + r) * p.num_heads + h) * kTcD + d] = __float2bfloat16(0.f);
        }
        return;
    }
    const int pos0 = ctx - nq;
    // KV tiles each Q tile reads (0 for a Q tile past the last query row)
    int ntq[kTcQT];
#pragma unroll
    for (int t = 0; t < kTcQT; ++t) {
        const int first = row0 + t * kTcRows;
        ntq[t] = first < nq ? (pos0 + min(first + kTcRows, nq) - 1) / kTcKeys + 1 : 0;
    }
    const int ntiles = ntq[kTcQT - 1] > ntq[0] ? ntq[kTcQT - 1] : ntq[0];
    const int last_pos = pos0 + min(row0 + kTcQT * kTcRows, nq) - 1;
    const int count_from = tile == 0 ? 0 : (pos0 + row0 - 1) / kBlockSize + 1;  // blocks first read here
    const int32_t* tab = p.block_tables + (size_t)s * p.max_blocks_per_seq;
    const int nblk_seq = (ctx + kBlockSize - 1) / kBlockSize;

    // ---- TMEM: 512 columns
    if (warp == kMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp == kProducer) {
        // ================= producer =================
        if (lane == 0) {
            // rows past total_q read zeros (the tensor map ends there)
            mbar_arrive_expect_tx(q_full, kTcQT * kTcQBytes);
            for (int t = 0; t < kTcQT; ++t) {
                tma_load_3d(base + kTcQ + t * kTcQBytes, &tmQ, 0, h, qs0 + row0 + t * kTcRows, q_full);
                tma_load_3d(base + kTcQ + t * kTcQBytes + kTcQChunk, &tmQ, 64, h, qs0 + row0 + t * kTcRows, q_full);
            }
        }
        {
            // E4M3 tiles: TMA into a 2-deep staging ring, up to two tiles ahead of the
            // converters (16-slot x 1-head x 128-byte boxes, 128-byte swizzle)
            bool ok = true;
            for (int j = 0; j < ntiles && !*abort_flag; ++j) {
                const int jb = j * kTcBlocks + (lane & (kTcBlocks - 1));
                int id = -1;
                if (lane < kTcBlocks && jb < nblk_seq) id = __ldg(tab + jb);
                const bool load = lane < kTcBlocks && jb < nblk_seq && id >= 0 && id < p.num_blocks;
                if (lane < kTcBlocks && jb < nblk_seq && !load && h == 0 && jb >= count_from &&
                    jb <= last_pos / kBlockSize)
                    count_error(p.err);
                const unsigned loaded = __ballot_sync(0xffffffffu, load);
                if (j >= 2) {
                    bool free_slot = true;
                    if (lane == 0) free_slot = mbar_wait_bounded(stg_empty + 8 * (j & 1), ((j >> 1) - 1) & 1);
                    if (!(ok = __shfl_sync(0xffffffffu, free_slot, 0))) break;
                }
                const uint32_t kst = base + kTcStg + (j & 1) * 2 * kTcStgBytes, vst = kst + kTcStgBytes;
                const uint32_t bar = stg_full + 8 * (j & 1);
                if (lane == 0) mbar_arrive_expect_tx(bar, __popc(loaded) * 2 * (kBlockSize * 128));
                __syncwarp();
                if (load) {
                    tma_load_3d(kst + lane * kBlockSize * 128, &tmK, 0, kvh, id * kBlockSize, bar);
                    tma_load_3d(vst + lane * kBlockSize * 128, &tmV, 0, kvh, id * kBlockSize, bar);
                }
            }
            if (!ok && lane == 0) {
                count_error(p.err);
                atomicExch(&abort_sh, 1);
            }
        }
    } else if (warp >= kConv0) {
        // ================= converters: warp kConv0 + b owns block b of each tile =================
        // The E4M3 codes of the block's 16 K and V rows become f16 in the swizzled
        // operand layout.  Lane order: item i = (row pair i >> 4, half (i >> 3) & 1,
        // 16-code chunk i & 7); a pair's rows split their chunks 0-3 / 4-7 between the
        // halves, so that each 8-lane quarter of a 16-byte access reads and writes 8
        // distinct bank groups.
        const int b = warp - kConv0;
        bool ok = true;
        for (int j = 0; j < ntiles && !*abort_flag; ++j) {
            const int st = j % kTcStages, round = j / kTcStages;
            const int jb = j * kTcBlocks + b;
            int id = -1;
            if (jb < nblk_seq) id = __ldg(tab + jb);
            const bool blk = jb < nblk_seq && id >= 0 && id < p.num_blocks;  // warp-uniform
            bool go = true;
            if (lane == 0) {
                if (round > 0) go = mbar_wait_bounded(kv_empty + 8 * st, (round - 1) & 1);
                if (go) go = mbar_wait_bounded(stg_full + 8 * (j & 1), (j >> 1) & 1);
            }
            if (!(ok = __shfl_sync(0xffffffffu, go, 0))) break;
            const uint32_t kst = base + kTcStg + (j & 1) * 2 * kTcStgBytes, vst = kst + kTcStgBytes;
            const uint32_t kdst = base + kTcKV + st * 2 * kTcKVBytes, vdst = kdst + kTcKVBytes;
            const int tail_from = ctx - j * kTcKeys;  // V rows from here on hold no token
            uint32_t src[4], dlo[4], dhi[4];
            int row[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = u * 32 + lane, c = i & 7;
                const int r = b * kBlockSize + 2 * (i >> 4) + ((c >> 2) ^ ((i >> 3) & 1));
                row[u] = r;
                src[u] = (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
                // f16 pieces 2c and 2c+1 of the row: column chunk c >> 2, slots swizzled by the row
                dlo[u] = (uint32_t)((c >> 2) * kTcKVChunk + r * 128 + ((((2 * c) & 7) ^ (r & 7)) << 4));
                dhi[u] = (uint32_t)((c >> 2) * kTcKVChunk + r * 128 + ((((2 * c + 1) & 7) ^ (r & 7)) << 4));
            }
            if (blk) {
                uint4 kc[4], vc[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(kc[u].x), "=r"(kc[u].y), "=r"(kc[u].z), "=r"(kc[u].w)
                                 : "r"(kst + src[u]));
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(vc[u].x), "=r"(vc[u].y), "=r"(vc[u].z), "=r"(vc[u].w)
                                 : "r"(vst + src[u]));
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint4 lo, hi;
                    e4m3x16_to_f16(kc[u], lo, hi);
                    st_shared_v4(kdst + dlo[u], lo);
                    st_shared_v4(kdst + dhi[u], hi);
                    if (row[u] < tail_from) {
                        e4m3x16_to_f16(vc[u], lo, hi);
                    } else {  // a slot past the context: no token, V stays zero
                        lo = make_uint4(0u, 0u, 0u, 0u);
                        hi = lo;
                    }
                    st_shared_v4(vdst + dlo[u], lo);
                    st_shared_v4(vdst + dhi[u], hi);
                }
            } else {
                // a block not loaded: its K stays as it was (its scores are masked), V is zero
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    st_shared_v4(vdst + dlo[u], z);
                    st_shared_v4(vdst + dhi[u], z);
                }
            }
            fence_proxy_async_smem();  // generic stores read by the tensor core; staging reads before TMA reuse
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(stg_empty + 8 * (j & 1));
                mbar_arrive(kv_full + 8 * st);
                mbar_arrive(v_ready + 8 * st);
            }
        }
        if (!ok && lane == 0) {
            count_error(p.err);
            atomicExch(&abort_sh, 1);
        }
    } else if (warp == kMma) {
        // ================= MMA issuer (warp-uniform, one elected lane issues) =================
        // S_t(0), S_t(1) first; then per KV tile j: PV_0(j), S_0(j+2), PV_1(j), S_1(j+2).
        // The scores are double-buffered, so a Q tile's softmax of tile j+1 runs while
        // the tensor core does PV(j) and S(j+2)
        const uint32_t idesc_s = instr_desc_16(kTcRows, kTcKeys, false, true);
        const uint32_t idesc_o = instr_desc_16(kTcRows, kTcD, true, true);
        // descriptors of an operand's first k-step; a k-step adds its byte offset >> 4 to
        // the start-address field (all of shared memory is below 2^18 bytes: no carry)
        const uint64_t dq0 = smem_desc(base + kTcQ, 16, 1024);
        const uint64_t dkv0 = smem_desc(base + kTcKV, 16, 1024);
        const uint64_t dvv0 = smem_desc(base + kTcKV + kTcKVBytes, kTcKVChunk, 1024);
        auto wait_all = [&](uint32_t bar, uint32_t parity) {
            return __all_sync(kFull, mbar_wait_bounded(bar, parity));
        };
        auto issue_s = [&](int t, int j) {
            tc_fence_after();
            const uint64_t dk = dkv0 + (uint64_t)(((j % kTcStages) * 2 * kTcKVBytes) >> 4);
            const uint64_t dq = dq0 + (uint64_t)((t * kTcQBytes) >> 4);
            const int sb = 2 * t + (j & 1);
#pragma unroll
            for (int ks = 0; ks < kTcD / 16; ++ks)
                umma_ss_e(tmem + kTcSCol + sb * kTcKeys, dq + (uint64_t)((((ks >> 2) * kTcQChunk) + (ks & 3) * 32) >> 4),
                          dk + (uint64_t)((((ks >> 2) * kTcKVChunk) + (ks & 3) * 32) >> 4), idesc_s, ks > 0 ? 1u : 0u);
            umma_commit_e(s_full + 8 * sb);
        };
        auto issue_pv = [&](int t, int j, bool pre) -> bool {
            if (!pre && !wait_all(p_full + 8 * (2 * t + (j & 1)), (j >> 1) & 1)) return false;
            if (!pre && !wait_all(v_ready + 8 * (j % kTcStages), (j / kTcStages) & 1)) return false;
            tc_fence_after();
            const uint64_t dv = dvv0 + (uint64_t)(((j % kTcStages) * 2 * kTcKVBytes) >> 4);
            // P_t(j) from TMEM over its score buffer: 16 keys = 8 columns per k-step.  The
            // S_t(j+2) product, issued after this one, overwrites them: the tensor core
            // runs one thread's products in issue order.
            const int sb = 2 * t + (j & 1);
#pragma unroll
            for (int ks = 0; ks < kTcKeys / 16; ++ks)
                umma_ts_e(tmem + kTcOCol + t * kTcD, tmem + kTcSCol + sb * kTcKeys + ks * 8,
                          dv + (uint64_t)((ks * 16 * 128) >> 4), idesc_o, (j > 0 || ks > 0) ? 1u : 0u);
            umma_commit_e(pv_done + 8 * sb);
            return true;
        };
        bool alive = wait_all(q_ready, 0);
        for (int j = 0; j < 2 && j < ntiles && alive; ++j) {
            alive = wait_all(kv_full + 8 * (j % kTcStages), (j / kTcStages) & 1);
            for (int t = 0; t < kTcQT && alive; ++t)
                if (j < ntq[t]) issue_s(t, j);
        }
        for (int j = 0; j < ntiles && alive; ++j) {
            if (__any_sync(kFull, *abort_flag != 0)) break;
            // every condition of this tile tested at once (their latencies overlap);
            // the ordered bounded waits only when one is not met yet
            bool pre = mbar_try_wait(v_ready + 8 * (j % kTcStages), (j / kTcStages) & 1);
            if (j < ntq[0]) pre = mbar_try_wait(p_full + 8 * (j & 1), (j >> 1) & 1) && pre;
            if (j < ntq[1]) pre = mbar_try_wait(p_full + 8 * (2 + (j & 1)), (j >> 1) & 1) && pre;
            if (j + 2 < ntiles) pre = mbar_try_wait(kv_full + 8 * ((j + 2) % kTcStages), ((j + 2) / kTcStages) & 1) && pre;
            pre = __all_sync(kFull, pre);
            for (int t = 0; t < kTcQT && alive; ++t) {
                if (j < ntq[t]) alive = issue_pv(t, j, pre);
                if (alive && j + 2 < ntq[t]) {
                    alive = pre || wait_all(kv_full + 8 * ((j + 2) % kTcStages), ((j + 2) / kTcStages) & 1);
                    if (alive) issue_s(t, j + 2);
                }
            }
            if (alive) umma_commit_e(kv_empty + 8 * (j % kTcStages));
        }
        if (!alive && lane == 0) {
            count_error(p.err);
            atomicExch(&abort_sh, 1);
        }
    } else {
        // ================= softmax: warpgroup t = Q tile t, thread = query row =================
        const int t = warp >> 2;
        const int r = threadIdx.x & 127;             // TMEM lane
        const int qrow = row0 + t * kTcRows + r;     // query row in the sequence
        const int qpos = pos0 + qrow;
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t o_addr = lane_addr + kTcOCol + t * kTcD;
        float m_ref = -INFINITY, l = 0.f;
        bool alive = true;
        const int nt = ntq[t];
        float row_scale = p.score_scale;  // this row's scores -> base-2 units
        {
            // The products run in f16 (an E4M3 code is exact there), and f16 does not
            // span bf16's range: each thread turns its own query row of the Q tile
            // into f16 in place after multiplying it by a power of two 2^e that puts
            // the row's largest magnitude in [2^14, 2^15) (exact; entries down to
            // 2^-28 of it keep all their bf16 bits), and takes 2^-e into its score
            // scale.  Row r of the tile is 128 bytes in each 64-column half, its
            // 16-byte chunks permuted by (r & 7): 8 consecutive rows touch 8
            // distinct bank groups.
            const bool landed = mbar_wait_bounded(q_full, 0);
            if (__all_sync(0xffffffffu, landed)) {
                const uint32_t qt = base + kTcQ + t * kTcQBytes;
                auto chunk_addr = [&](int c) {  // c = 0..15: half c / 8, chunk c % 8 of row r
                    return qt + (c >> 3) * (kTcRows * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
                };
                uint4 v[16];  // the row, one pass: loads, maximum, conversion, stores
                uint32_t m2 = 0;  // two 16-bit maxima of |x| as bits (sign cleared)
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    v[c] = ld_shared_v4(chunk_addr(c));
                    m2 = __vmaxu2(m2, __vmaxu2(__vmaxu2(v[c].x & 0x7FFF7FFFu, v[c].y & 0x7FFF7FFFu),
                                               __vmaxu2(v[c].z & 0x7FFF7FFFu, v[c].w & 0x7FFF7FFFu)));
                }
                const uint32_t amax_bits = max(m2 & 0xFFFFu, m2 >> 16);
                // e = 14 - floor(log2 max|q|) within [-126, 126]; an all-zero row keeps e = 0
                const int ex = amax_bits != 0 ? (int)(amax_bits >> 7) - 127 : 14;
                const int e = min(max(14 - ex, -126), 126);
                const float up = __uint_as_float((uint32_t)(127 + e) << 23);
                row_scale = __uint_as_float((uint32_t)(127 - e) << 23) * p.score_scale;
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    uint4 w = v[c];
                    w.x = bf16x2_to_f16x2_scaled(w.x, up);
                    w.y = bf16x2_to_f16x2_scaled(w.y, up);
                    w.z = bf16x2_to_f16x2_scaled(w.z, up);
                    w.w = bf16x2_to_f16x2_scaled(w.w, up);
                    st_shared_v4(chunk_addr(c), w);
                }
                fence_proxy_async_smem();  // read by the tensor core
                __syncwarp();
                if (lane == 0) mbar_arrive(q_ready);
            } else {
                alive = false;
            }
        }
        // validity of the blocks this CTA reads, once, into shared memory (both
        // warpgroups together; the named barrier counts their 256 threads only)
        const int nblk_cta = min(nblk_seq, (last_pos / kBlockSize) + 1);
        const bool bits_in_smem = nblk_cta <= 32 * kTcOkWords;
        if (bits_in_smem) {
            for (int w = threadIdx.x; w < kTcOkWords; w += 256) ok_bits[w] = 0u;
            asm volatile("bar.sync 1, 256;" ::: "memory");
            for (int b = threadIdx.x; b < nblk_cta; b += 256) {
                const int id = __ldg(tab + b);
                if (id >= 0 && id < p.num_blocks) atomicOr(&ok_bits[b >> 5], 1u << (b & 31));
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
        }
        for (int j = 0; j < nt && alive; ++j) {
            if (*abort_flag) {
                alive = false;
                break;
            }
            // blocks of this tile that hold tokens (in the table, id in range)
            unsigned okmask = 0;
            if (bits_in_smem) {
                okmask = (ok_bits[(j * kTcBlocks) >> 5] >> ((j * kTcBlocks) & 31)) & ((1u << kTcBlocks) - 1u);
            } else {
#pragma unroll
                for (int b = 0; b < kTcBlocks; ++b) {
                    const int jb = j * kTcBlocks + b;
                    const int id = jb < nblk_seq ? __ldg(tab + jb) : -1;
                    if (id >= 0 && id < p.num_blocks) okmask |= 1u << b;
                }
            }
            const int sb = 2 * t + (j & 1);
            const uint32_t s_addr = lane_addr + kTcSCol + sb * kTcKeys;
            const bool w1 = mbar_wait_bounded(s_full + 8 * sb, (j >> 1) & 1);
            if (!__all_sync(0xffffffffu, w1)) {
                alive = false;
                break;
            }
            tc_fence_after();
            float x[kTcKeys];
#pragma unroll
            for (int c2 = 0; c2 < kTcKeys / 32; ++c2) {
                float v[32];
                tmem_ld32(s_addr + 32 * c2, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) x[32 * c2 + i] = v[i];
            }
            tmem_wait_ld();
            const int k0 = j * kTcKeys;
            if (k0 + kTcKeys - 1 <= qpos && okmask == (1u << kTcBlocks) - 1u) {
#pragma unroll
                for (int c = 0; c < kTcKeys; ++c) x[c] *= row_scale;
            } else {
#pragma unroll
                for (int c = 0; c < kTcKeys; ++c) {
                    const bool valid = k0 + c <= qpos && ((okmask >> (c >> 4)) & 1u);
                    x[c] = valid ? x[c] * row_scale : -INFINITY;
                }
            }
            // max as 8 independent chains, then a tree (short dependency chains)
            float mx8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mx8[i] = x[i];
#pragma unroll
            for (int c = 8; c < kTcKeys; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], x[c]);
            const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                   fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            // the reference max moves only when a score exceeds it by more than 2^8
            float alpha = 1.f;
            const bool move = mx > m_ref + kRescaleThreshold || m_ref == -INFINITY;
            const float m_new = move ? mx : m_ref;
            if (move && m_ref != -INFINITY) alpha = fast_exp2(m_ref - m_new);
            const float mu = m_new == -INFINITY ? 0.f : m_new;
            // P row as 16-bit pairs
            uint32_t pw[kTcKeys / 2];
            float sum8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int e = 0; e < kTcKeys / 2; ++e) {
                const float p0 = fast_exp2(x[2 * e] - mu), p1 = fast_exp2(x[2 * e + 1] - mu);
                sum8[e & 7] += p0 + p1;
                pw[e] = pack_f16x2(p0, p1);
            }
            const float sum = ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
            // a moved reference max rescales O, once PV(j-1) has landed in it (PV(j+1), the
            // next on that barrier, waits for P(j+1): the barrier is at most one phase on)
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                const bool w2 = mbar_wait_bounded(pv_done + 8 * (2 * t + ((j - 1) & 1)), ((j - 1) >> 1) & 1);
                if (!__all_sync(0xffffffffu, w2)) {
                    alive = false;
                    break;
                }
                tc_fence_after();
#pragma unroll 1
                for (int c4 = 0; c4 < kTcD / 32; ++c4) {
                    float v[32];
                    tmem_ld32(o_addr + 32 * c4, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= alpha;
                    tmem_st32(o_addr + 32 * c4, v);
                }
                tmem_wait_st();
            }
            l = l * alpha + sum;
            m_ref = m_new;
            // P row into TMEM over the first 32 columns of the scores just read
            {
                float pf[kTcKeys / 2];
#pragma unroll
                for (int e = 0; e < kTcKeys / 2; ++e) pf[e] = __uint_as_float(pw[e]);
                tmem_st32(s_addr, pf);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full + 8 * sb);
        }
        if (!alive && lane == 0) {
            count_error(p.err);
            atomicExch(&abort_sh, 1);
        }
        // epilogue: wait for the last PV, normalise and store the row
        if (alive && nt > 0 && !*abort_flag) {
            // PV(nt-1) is the last product into O; its commit covers every earlier one
            const bool w3 = mbar_wait_bounded(pv_done + 8 * (2 * t + ((nt - 1) & 1)), ((nt - 1) >> 1) & 1);
            if (__all_sync(0xffffffffu, w3)) {
                tc_fence_after();
                const float inv = l > 0.f ? p.out_scale / l : 0.f;
                const bool store = qrow < nq;
                __nv_bfloat16* out = p.out + ((size_t)(qs0 + (store ? qrow : 0)) * p.num_heads + h) * kTcD;
#pragma unroll 1
                for (int c4 = 0; c4 < kTcD / 32; ++c4) {
                    float v[32];
                    tmem_ld32(o_addr + 32 * c4, v);
                    tmem_wait_ld();
                    if (store) {
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            uint4 u;
                            u.x = pack_bf16x2(v[i] * inv, v[i + 1] * inv);
                            u.y = pack_bf16x2(v[i + 2] * inv, v[i + 3] * inv);
                            u.z = pack_bf16x2(v[i + 4] * inv, v[i + 5] * inv);
                            u.w = pack_bf16x2(v[i + 6] * inv, v[i + 7] * inv);
                            *reinterpret_cast<uint4*>(out + 32 * c4 + i) = u;
                        }
                    }
                }
            } else if (lane == 0) {
                count_error(p.err);
                atomicExch(&abort_sh, 1);
            }
        }
    }

    // ---- every role is done with TMEM and the ring
    tc_fence_before();
    __syncthreads();
    if (warp == kMma) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

// Causal prompt pass over a bf16 cache with 128-key tiles.  One CTA per (sequence,
// 256 query rows = two Q tiles of 128, query head); twelve warps, of which warps 10
// and 11 only complete warpgroup 2 (warps 8-11), so that registers can move between
// warpgroups: launched at 168 per thread (65,536 / 384), warpgroup 2 gives up to 80
// and the softmax warpgroups take 200 (2 x 128 x 200 + 128 x 80 = 61,440 <= 384 x 168;
// 200 registers hold a row's 128 scores and its P without spills, where 168 spilled):
//  - warp 8 (producer): TMA-loads the two Q tiles once, then per 128-key tile the K
//    of 8 table blocks into a 2-stage ring and their V into another (16-slot x
//    1-head x 128-byte boxes, 128-byte swizzle), zeroing the V rows that hold no
//    token of the context;
//  - warp 9 (MMA): runs warp-uniformly, one elected lane issuing.  Per KV tile j and
//    Q tile t: O_t += P_t(j) V(j) (P_t from TMEM), then S_t(j+1) = Q_t K(j+1)^T
//    (M = N = 128, K = 128) into the Q tile's one score buffer.  The tensor core runs
//    one thread's products in issue order, so S_t(j+1) overwrites P_t(j) only after
//    PV_t(j) has read it, and the commit that signals S_t(j+1) also covers PV_t(j).
//    While one Q tile's softmax runs, the tensor core does the other Q tile's PV and
//    next scores;
//  - warps 0-3 and 4-7 (softmax, one warpgroup per Q tile, thread r = query row r =
//    TMEM lane r): per KV tile loads the row's 128 scores, masks the causal boundary
//    and the blocks with no token, runs the online softmax in base 2 (the reference
//    max moves only when a score exceeds it by more than 2^8; O, complete up to the
//    previous tile when the scores land, is then rescaled in TMEM), writes P as bf16
//    pairs over the first 64 score columns, and finally normalises O and stores the
//    row.
__global__ void __launch_bounds__(384, 1)
    prefill_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
    extern __shared__ uint8_t smem_raw[];
    // k_full[2], k_empty[2], v_full[2], v_ready[2], v_empty[2], q_full, s_full[2], p_full[2], o_done[2]
    __shared__ __align__(8) uint64_t bars[2 * kWKStages + 3 * kWVStages + 1 + 3 * kTcQT];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    __shared__ uint32_t ok_bits[kTcOkWords];
    volatile int* abort_flag = &abort_sh;
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t k_full = smem_u32(&bars[0]), k_empty = k_full + 8 * kWKStages, v_full = k_empty + 8 * kWKStages,
                   v_ready = v_full + 8 * kWVStages, v_empty = v_ready + 8 * kWVStages, q_full = v_empty + 8 * kWVStages,
                   s_full = q_full + 8, p_full = s_full + 8 * kTcQT, o_done = p_full + 8 * kTcQT;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kProducer = 8, kMma = 9;
    constexpr uint32_t kFull = 0xffffffffu;

    // grid (head, 256-row tile, sequence): a sequence's CTAs run together (its K/V
    // stays in L2 for all its tiles and heads), its last rows (the most KV tiles)
    // first, so that each sequence's CTAs reach the SMs longest first and end short
    const int h = blockIdx.x, s = blockIdx.z, kvh = h / p.group;
    const int tile = gridDim.y - 1 - blockIdx.y;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kWKStages; ++i) {
            mbar_init(k_full + 8 * i, 1);
            mbar_init(k_empty + 8 * i, 1);
        }
        for (int i = 0; i < kWVStages; ++i) {
            mbar_init(v_full + 8 * i, 1);
            mbar_init(v_ready + 8 * i, 1);
            mbar_init(v_empty + 8 * i, 1);
        }
        mbar_init(q_full, 1);
        for (int t = 0; t < kTcQT; ++t) {
            mbar_init(s_full + 8 * t, 1);
            mbar_init(p_full + 8 * t, 4);
            mbar_init(o_done + 8 * t, 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kProducer && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();

    const int qs0 = p.query_start[s];
    const int nq = p.query_start[s + 1] - qs0;
    const int ctx = p.context_lens[s];
    const int row0 = tile * (kTcQT * kTcRows);
    if (row0 >= nq) return;  // the whole CTA leaves together, before TMEM allocation
    if (nq > ctx || ctx > p.max_blocks_per_seq * kBlockSize) {
        if (tile == 0 && h == 0 && threadIdx.x == 0) count_error(p.err);
        const int rows = min(kTcQT * kTcRows, nq - row0);
        for (int e = threadIdx.x; e < rows * kTcD; e += blockDim.x) {
            const int r = e / kTcD, d = e - r * kTcD;
            p.out[((size_t)(qs0 + row0 + r) * p.num_heads + h) * kTcD + d] = __float2bfloat16(0.f);
        }
        return;
    }
    const int pos0 = ctx - nq;
    int ntq[kTcQT];  // KV tiles each Q tile reads (0 for a Q tile past the last query row)
#pragma unroll
    for (int t = 0; t < kTcQT; ++t) {
        const int first = row0 + t * kTcRows;
        ntq[t] = first < nq ? (pos0 + min(first + kTcRows, nq) - 1) / kWKeys + 1 : 0;
    }
    const int ntiles = max(ntq[0], ntq[1]);
    const int last_pos = pos0 + min(row0 + kTcQT * kTcRows, nq) - 1;
    const int count_from = tile == 0 ? 0 : (pos0 + row0 - 1) / kBlockSize + 1;  // blocks first read here
    const int32_t* tab = p.block_tables + (size_t)s * p.max_blocks_per_seq;
    const int nblk_seq = (ctx + kBlockSize - 1) / kBlockSize;

    if (warp == kMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    // registers move from warpgroup 2 (producer, issuer, two idle warps) to the two
    // softmax warpgroups; each warpgroup's four warps run its setmaxnreg together
    if (warp >= 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 80;");
        if (warp == kProducer) {
            // ================= producer =================
            if (lane == 0) {
                mbar_arrive_expect_tx(q_full, kTcQT * kTcQBytes);
                for (int t = 0; t < kTcQT; ++t) {
                    tma_load_3d(base + t * kTcQBytes, &tmQ, 0, h, qs0 + row0 + t * kTcRows, q_full);
                    tma_load_3d(base + t * kTcQBytes + kTcQChunk, &tmQ, 64, h, qs0 + row0 + t * kTcRows, q_full);
                }
            }
            bool ok = true;
            for (int j = 0; j < ntiles && !*abort_flag; ++j) {
                // block ids of this tile: lanes 0..7; a block is loaded if it is in the table
                // and its id is in range
                const int jb = j * kWBlocks + (lane & (kWBlocks - 1));
                int id = -1;
                if (lane < kWBlocks && jb < nblk_seq) id = __ldg(tab + jb);
                const bool load = lane < kWBlocks && jb < nblk_seq && id >= 0 && id < p.num_blocks;
                if (lane < kWBlocks && jb < nblk_seq && !load && h == 0 && jb >= count_from && jb <= last_pos / kBlockSize)
                    count_error(p.err);
                const unsigned loaded = __ballot_sync(kFull, load);
                const int row = id * kBlockSize;
                const uint32_t off = lane * kBlockSize * 128;
                const uint32_t tx = __popc(loaded) * 2 * (kBlockSize * 128);
                // K of this tile into its ring slot, once the products that read the slot's
                // previous tile are done
                const int ks = j % kWKStages, kr = j / kWKStages;
                bool go = true;
                if (lane == 0 && kr > 0) go = mbar_wait_bounded(k_empty + 8 * ks, (kr - 1) & 1);
                if (!(ok = __shfl_sync(kFull, go, 0))) break;
                const uint32_t kdst = base + kWK + ks * kWTile;
                if (lane == 0) mbar_arrive_expect_tx(k_full + 8 * ks, tx);
                __syncwarp();
                if (load) {
                    tma_load_3d(kdst + off, &tmK, 0, kvh, row, k_full + 8 * ks);
                    tma_load_3d(kdst + kWChunk + off, &tmK, 64, kvh, row, k_full + 8 * ks);
                }
                // V likewise
                const int vs = j % kWVStages, vr = j / kWVStages;
                if (lane == 0 && vr > 0) go = mbar_wait_bounded(v_empty + 8 * vs, (vr - 1) & 1);
                if (!(ok = __shfl_sync(kFull, go, 0))) break;
                const uint32_t vdst = base + kWV + vs * kWTile;
                if (lane == 0) mbar_arrive_expect_tx(v_full + 8 * vs, tx);
                __syncwarp();
                if (load) {
                    tma_load_3d(vdst + off, &tmV, 0, kvh, row, v_full + 8 * vs);
                    tma_load_3d(vdst + kWChunk + off, &tmV, 64, kvh, row, v_full + 8 * vs);
                }
                // V rows with no token: whole blocks not loaded, and the slots past the context
                // in the sequence's last block (once it has landed)
                for (int b = 0; b < kWBlocks; ++b) {
                    if ((loaded >> b) & 1u) continue;
                    for (int i = lane; i < kBlockSize * 16; i += 32) {
                        const int r = b * kBlockSize + (i >> 4), c = i & 15;
                        const uint32_t a = vdst + (c >> 3) * kWChunk + r * 128 + ((c & 7) << 4);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0) : "memory");
                    }
                }
                const int jt = (ctx % kBlockSize) ? nblk_seq - 1 : -1;
                const int bt = jt - j * kWBlocks;
                if (bt >= 0 && bt < kWBlocks && ((loaded >> bt) & 1u)) {
                    bool landed = true;
                    if (lane == 0) landed = mbar_wait_bounded(v_full + 8 * vs, vr & 1);
                    if (!(ok = __shfl_sync(kFull, landed, 0))) break;
                    const int r0 = ctx % kBlockSize;
                    for (int i = lane; i < (kBlockSize - r0) * 16; i += 32) {
                        const int r = bt * kBlockSize + r0 + (i >> 4), c = i & 15;
                        const uint32_t a = vdst + (c >> 3) * kWChunk + r * 128 + ((c & 7) << 4);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0) : "memory");
                    }
                }
                fence_proxy_async_smem();  // these generic stores are read by the tensor core
                __syncwarp();
                if (lane == 0) mbar_arrive(v_ready + 8 * vs);
            }
            if (!ok && lane == 0) {
                count_error(p.err);
                atomicExch(&abort_sh, 1);
            }
        } else if (warp == kMma) {
            // ================= MMA issuer (warp-uniform) =================
            const uint32_t idesc_s = instr_desc_16(kTcRows, kWKeys, false, false);
            const uint32_t idesc_o = instr_desc_16(kTcRows, kTcD, true, false);
            // descriptors of an operand's first k-step; a k-step adds its byte offset >> 4 to
            // the start-address field (all of shared memory is below 2^18 bytes: no carry)
            const uint64_t dq0 = smem_desc(base, 16, 1024);
            const uint64_t dk0 = smem_desc(base + kWK, 16, 1024);
            const uint64_t dv0 = smem_desc(base + kWV, kWChunk, 1024);
            auto wait_all = [&](uint32_t bar, uint32_t parity) {
                return __all_sync(kFull, mbar_wait_bounded(bar, parity));
            };
            auto issue_s = [&](int t, int j) {
                tc_fence_after();
                const uint64_t dk = dk0 + (uint64_t)(((j % kWKStages) * kWTile) >> 4);
                const uint64_t dq = dq0 + (uint64_t)((t * kTcQBytes) >> 4);
    #pragma unroll
                for (int k = 0; k < kTcD / 16; ++k)
                    umma_ss_e(tmem + kWSCol + t * kWKeys, dq + (uint64_t)((((k >> 2) * kTcQChunk) + (k & 3) * 32) >> 4),
                              dk + (uint64_t)((((k >> 2) * kWChunk) + (k & 3) * 32) >> 4), idesc_s, k > 0 ? 1u : 0u);
                umma_commit_e(s_full + 8 * t);
            };
            auto issue_pv = [&](int t, int j) {
                tc_fence_after();
                const uint64_t dv = dv0 + (uint64_t)(((j % kWVStages) * kWTile) >> 4);
                // P_t(j) from TMEM over the Q tile's score buffer: 16 keys = 8 columns per k-step
    #pragma unroll
                for (int k = 0; k < kWKeys / 16; ++k)
                    umma_ts_e(tmem + t * kTcD, tmem + kWSCol + t * kWKeys + k * 8, dv + (uint64_t)((k * 16 * 128) >> 4),
                              idesc_o, (j > 0 || k > 0) ? 1u : 0u);
            };
            bool alive = wait_all(q_full, 0) && wait_all(k_full, 0);
            if (alive) {
                for (int t = 0; t < kTcQT; ++t)
                    if (ntq[t] > 0) issue_s(t, 0);
                umma_commit_e(k_empty);
            }
            for (int j = 0; j < ntiles && alive; ++j) {
                if (__any_sync(kFull, *abort_flag != 0)) break;
                bool v_in = false, k_in = false;
                for (int t = 0; t < kTcQT && alive; ++t) {
                    if (j < ntq[t]) {
                        alive = wait_all(p_full + 8 * t, j & 1);
                        // V landed (its own copy barrier) and its empty rows zeroed (producer)
                        if (alive && !v_in)
                            alive = wait_all(v_full + 8 * (j % kWVStages), (j / kWVStages) & 1) &&
                                    wait_all(v_ready + 8 * (j % kWVStages), (j / kWVStages) & 1);
                        v_in = true;
                        if (!alive) break;
                        issue_pv(t, j);
                        if (j == ntq[t] - 1) umma_commit_e(o_done + 8 * t);
                    }
                    if (j + 1 < ntq[t]) {
                        if (!k_in) alive = wait_all(k_full + 8 * ((j + 1) % kWKStages), ((j + 1) / kWKStages) & 1);
                        k_in = true;
                        if (!alive) break;
                        issue_s(t, j + 1);
                    }
                }
                if (!alive) break;
                if (j + 1 < ntiles) umma_commit_e(k_empty + 8 * ((j + 1) % kWKStages));
                umma_commit_e(v_empty + 8 * (j % kWVStages));
            }
            if (!alive && lane == 0) {
                count_error(p.err);
                atomicExch(&abort_sh, 1);
            }
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 200;");
        // ================= softmax: warpgroup t = Q tile t, thread = query row =================
        const int t = warp >> 2;
        const int r = threadIdx.x & 127;
        const int qrow = row0 + t * kTcRows + r;
        const int qpos = pos0 + qrow;
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t o_addr = lane_addr + t * kTcD;
        const uint32_t s_addr = lane_addr + kWSCol + t * kWKeys;
        float m_ref = -INFINITY, l = 0.f;
        bool alive = true;
        const int nt = ntq[t];
        // scores x * score_scale: a negative scale is taken as |scale| on -x
        const bool neg = p.score_scale < 0.f;
        const float sc = fabsf(p.score_scale);
        const int nblk_cta = min(nblk_seq, (last_pos / kBlockSize) + 1);
        const bool bits_in_smem = nblk_cta <= 32 * kTcOkWords;
        if (bits_in_smem) {
            for (int w = threadIdx.x; w < kTcOkWords; w += 256) ok_bits[w] = 0u;
            asm volatile("bar.sync 1, 256;" ::: "memory");
            for (int b = threadIdx.x; b < nblk_cta; b += 256) {
                const int id = __ldg(tab + b);
                if (id >= 0 && id < p.num_blocks) atomicOr(&ok_bits[b >> 5], 1u << (b & 31));
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
        }
        for (int j = 0; j < nt && alive; ++j) {
            if (*abort_flag) {
                alive = false;
                break;
            }
            unsigned okmask = 0;  // blocks of this tile that hold tokens
            if (bits_in_smem) {
                okmask = (ok_bits[(j * kWBlocks) >> 5] >> ((j * kWBlocks) & 31)) & ((1u << kWBlocks) - 1u);
            } else {
#pragma unroll
                for (int b = 0; b < kWBlocks; ++b) {
                    const int jb = j * kWBlocks + b;
                    const int id = jb < nblk_seq ? __ldg(tab + jb) : -1;
                    if (id >= 0 && id < p.num_blocks) okmask |= 1u << b;
                }
            }
            const bool w1 = mbar_wait_bounded(s_full + 8 * t, j & 1);
            if (!__all_sync(kFull, w1)) {
                alive = false;
                break;
            }
            tc_fence_after();
            float x[kWKeys];
#pragma unroll
            for (int c4 = 0; c4 < kWKeys / 32; ++c4) {
                uint32_t u[32];
                tmem_ld32_u(s_addr + 32 * c4, u);
#pragma unroll
                for (int i = 0; i < 32; ++i) x[32 * c4 + i] = __uint_as_float(u[i]);
            }
            tmem_wait_ld();
            if (neg) {
#pragma unroll
                for (int c = 0; c < kWKeys; ++c) x[c] = -x[c];
            }
            const int k0 = j * kWKeys;
            const bool full = k0 + kWKeys - 1 <= qpos && okmask == (1u << kWBlocks) - 1u;
            if (!full) {
#pragma unroll
                for (int c = 0; c < kWKeys; ++c) {
                    const bool valid = k0 + c <= qpos && ((okmask >> (c >> 4)) & 1u);
                    x[c] = valid ? x[c] : -INFINITY;
                }
            }
            // the row's largest score: four chains of three-input maxima
            float m4[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
            for (int c = 4; c < kWKeys; c += 8) {
                m4[0] = max3(m4[0], x[c], x[c + 1]);
                m4[1] = max3(m4[1], x[c + 2], x[c + 3]);
                m4[2] = max3(m4[2], x[c + 4], x[c + 5]);
                m4[3] = max3(m4[3], x[c + 6], x[c + 7]);
            }
            const float mraw = max3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
            const float mx = mraw == -INFINITY ? -INFINITY : mraw * sc;  // no -inf * 0
            // the reference max moves only when a score exceeds it by more than 2^8
            float alpha = 1.f;
            if (mx > m_ref + kRescaleThreshold || m_ref == -INFINITY) {
                if (m_ref != -INFINITY) alpha = fast_exp2(m_ref - mx);
                m_ref = mx;
            }
            // O is complete up to the previous tile (its product preceded these scores)
            if (j > 0 && __any_sync(kFull, alpha != 1.f)) {
#pragma unroll 1
                for (int c4 = 0; c4 < kTcD / 32; ++c4) {
                    float v[32];
                    tmem_ld32(o_addr + 32 * c4, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= alpha;
                    tmem_st32(o_addr + 32 * c4, v);
                }
                tmem_wait_st();
            }
            const float mu = m_ref == -INFINITY ? 0.f : m_ref;
            const uint64_t sc2 = f2(sc, sc), nmu2 = f2(-mu, -mu);
            uint32_t pf[kWKeys / 2];
            const float sum = __all_sync(kFull, full) ? row_probs<false>(x, sc2, nmu2, 0, 0u, pf)
                                   : row_probs<true>(x, sc2, nmu2, qpos - k0, okmask, pf);
            l = l * alpha + sum;
            tmem_st32(s_addr, reinterpret_cast<const float(&)[32]>(pf[0]));
            tmem_st32(s_addr + 32, reinterpret_cast<const float(&)[32]>(pf[32]));
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full + 8 * t);
        }
        if (!alive && lane == 0) {
            count_error(p.err);
            atomicExch(&abort_sh, 1);
        }
        if (alive && nt > 0 && !*abort_flag) {
            const bool w3 = mbar_wait_bounded(o_done + 8 * t, 0);
            if (__all_sync(kFull, w3)) {
                tc_fence_after();
                const float inv = l > 0.f ? p.out_scale / l : 0.f;
                const bool store = qrow < nq;
                __nv_bfloat16* out = p.out + ((size_t)(qs0 + (store ? qrow : 0)) * p.num_heads + h) * kTcD;
#pragma unroll 1
                for (int c4 = 0; c4 < kTcD / 32; ++c4) {
                    float v[32];
                    tmem_ld32(o_addr + 32 * c4, v);
                    tmem_wait_ld();
                    if (store) {
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            uint4 u;
                            u.x = pack_bf16x2(v[i] * inv, v[i + 1] * inv);
                            u.y = pack_bf16x2(v[i + 2] * inv, v[i + 3] * inv);
                            u.z = pack_bf16x2(v[i + 4] * inv, v[i + 5] * inv);
                            u.w = pack_bf16x2(v[i + 6] * inv, v[i + 7] * inv);
                            *reinterpret_cast<uint4*>(out + 32 * c4 + i) = u;
                        }
                    }
                }
            } else if (lane == 0) {
                count_error(p.err);
                atomicExch(&abort_sh, 1);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMma) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

cudaError_t launch_prefill_tc(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                              const PrefillParams& p, bool fp8, int max_query_len, cudaStream_t stream) {
    const int tiles = (max_query_len + kTcQT * kTcRows - 1) / (kTcQT * kTcRows);
    const dim3 grid(p.num_heads, tiles, p.num_seqs);
    if (fp8) {
        const int smem = kTcSmemFp8 + 1024;
        cudaError_t e = cudaFuncSetAttribute(prefill_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        return launch_pdl(prefill_fp8_kernel, grid, dim3(448), smem, stream, tmQ, tmK, tmV, p);
    }
    const int smem = kWSmem + 1024;
    cudaError_t e = cudaFuncSetAttribute(prefill_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(prefill_bf16_kernel, grid, dim3(384), smem, stream, tmQ, tmK, tmV, p);
}

}  // namespace pkv
