// prefill_tc.cu -- causal multi-token paged attention on the 5th-generation
// tensor cores (tcgen05): same result as prefill.cu's kernel.
//
// What it computes: sequence s has nq new query tokens, the last nq of its
// context_len tokens (K/V already in the pool); query i at position
// p = context_len - nq + i attends to every token t <= p through the block table
// (iplexlaw.co.kr, logical vs physical order; gyaansetu.com, what the KV cache
// holds).
//
// One CTA per (sequence, 128 query rows, query head); six warps:
//  - warp 4 (producer): TMA-loads the Q tile once and, per 128-key tile, the K
//    and V of 8 blocks of the table (16-slot x 1-head x 128-byte boxes, 128-byte
//    swizzle) into a 2-stage ring; V rows that hold no token of the context
//    (past its end, or a block past the table or with a bad id) are zeroed in
//    shared memory, so that a zero probability never meets a NaN there;
//  - warp 5 (MMA): one thread issues tcgen05.mma: S = Q K^T (M=128, N=128,
//    K=128, bf16 -> fp32) into one of two TMEM buffers, then O += P V (P from
//    shared memory, V MN-major) into a TMEM accumulator; tcgen05.commit signals
//    mbarriers; the warp allocates and frees the 512 TMEM columns;
//  - warps 0-3 (softmax): thread r owns query row r (TMEM lane r): loads its
//    128 scores with tcgen05.ld, applies the causal mask, runs the online
//    softmax in base 2 (the reference max moves only when a score exceeds it by
//    more than 2^8, then O is rescaled in TMEM), writes P as bf16 into the
//    swizzled K-major layout the PV MMA reads, and finally normalises O and
//    stores the rows.
// S for tile j+1 is computed while the softmax works on tile j.
#include "pkv_common.cuh"

namespace pkv {

namespace {

constexpr int kTcRows = 128;                   // query rows per CTA (MMA M)
constexpr int kTcKeys = 128;                   // keys per tile (MMA N of S, K of PV)
constexpr int kTcD = 128;                      // head_dim
constexpr int kTcChunk = kTcRows * 128;        // one 64-element column chunk of a 128-row operand: 16 KB
constexpr int kTcOperand = 2 * kTcChunk;       // 128 rows x 128 bf16: 32 KB
constexpr int kTcStages = 2;
// shared memory layout (offsets from a 1024-aligned base)
constexpr int kTcQ = 0;
constexpr int kTcP = kTcQ + kTcOperand;
constexpr int kTcKV = kTcP + kTcOperand;       // stage st: K at kTcKV + st*2*kTcOperand, V after it
constexpr int kTcSmem = kTcKV + kTcStages * 2 * kTcOperand;  // 192 KB
constexpr float kRescaleThreshold = 8.f;       // log2 of the largest factor p may exceed 1 by

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

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator, M x N.
__host__ __device__ constexpr uint32_t instr_desc_bf16(int M, int N, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_ss(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"((uint32_t)accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
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

}  // namespace

__global__ void __launch_bounds__(192, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
    extern __shared__ uint8_t smem_raw[];
    // barriers: kv_full[2], kv_empty[2], q_full, s_full[2], p_full, pv_done, v_ready[2]
    __shared__ __align__(8) uint64_t bars[12];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    volatile int* abort_flag = &abort_sh;
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t b0 = smem_u32(&bars[0]);
    const uint32_t kv_full = b0, kv_empty = b0 + 16, q_full = b0 + 32, s_full = b0 + 40, p_full = b0 + 56,
                   pv_done = b0 + 64, v_ready = b0 + 72;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int s = blockIdx.y, h = blockIdx.z, kvh = h / p.group;
    const int tile = gridDim.x - 1 - blockIdx.x;
    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        mbar_init(kv_full + 8, 1);
        mbar_init(kv_empty, 1);
        mbar_init(kv_empty + 8, 1);
        mbar_init(q_full, 1);
        mbar_init(s_full, 1);
        mbar_init(s_full + 8, 1);
        mbar_init(p_full, 4);
        mbar_init(pv_done, 1);
        mbar_init(v_ready, 1);
        mbar_init(v_ready + 8, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 4 && lane == 0) {
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
    const int row0 = tile * kTcRows;
    if (row0 >= nq) return;  // the whole CTA leaves together, before TMEM allocation
    if (nq > ctx || ctx > p.max_blocks_per_seq * kBlockSize) {
        if (tile == 0 && h == 0 && threadIdx.x == 0) count_error(p.err);
        const int rows = min(kTcRows, nq - row0);
        for (int e = threadIdx.x; e < rows * kTcD; e += blockDim.x) {
            const int r = e / kTcD, d = e - r * kTcD;
            p.out[((size_t)(qs0 + row0 + r) * p.num_heads + h) * kTcD + d] = __float2bfloat16(0.f);
        }
        return;
    }
    const int pos0 = ctx - nq;
    const int last_row = min(row0 + kTcRows, nq) - 1;
    const int last_pos = pos0 + last_row;
    const int ntiles = last_pos / kTcKeys + 1;
    const int count_from = tile == 0 ? 0 : (pos0 + row0 - 1) / kBlockSize + 1;  // blocks first read here
    const int32_t* tab = p.block_tables + (size_t)s * p.max_blocks_per_seq;
    const int nblk_seq = (ctx + kBlockSize - 1) / kBlockSize;

    // ---- TMEM: 512 columns (S buffers at 0 and 128, O at 256)
    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp == 4) {
        // ================= producer =================
        if (lane == 0) {
            mbar_arrive_expect_tx(q_full, kTcOperand);
            // rows past total_q read zeros (the tensor map ends there)
            tma_load_3d(base + kTcQ, &tmQ, 0, h, qs0 + row0, q_full);
            tma_load_3d(base + kTcQ + kTcChunk, &tmQ, 64, h, qs0 + row0, q_full);
        }
        for (int j = 0; j < ntiles && !*abort_flag; ++j) {
            const int st = j % kTcStages, round = j / kTcStages;
            // block ids of this tile: lanes 0..7; a block is loaded if it is in the table
            // and its id is in range
            const int jb = j * 8 + (lane & 7);
            int id = -1;
            if (lane < 8 && jb < nblk_seq) id = __ldg(tab + jb);
            const bool load = lane < 8 && jb < nblk_seq && id >= 0 && id < p.num_blocks;
            if (lane < 8 && jb < nblk_seq && !load && h == 0 && jb >= count_from && jb <= last_pos / kBlockSize)
                count_error(p.err);
            const unsigned loaded = __ballot_sync(0xffffffffu, load);
            bool go = true;
            if (lane == 0 && round > 0) go = mbar_wait_bounded(kv_empty + 8 * st, (round - 1) & 1);
            go = __shfl_sync(0xffffffffu, go, 0);
            if (!go) {
                if (lane == 0) {
                    count_error(p.err);
                    atomicExch(&abort_sh, 1);
                }
                break;
            }
            const uint32_t kdst = base + kTcKV + st * 2 * kTcOperand, vdst = kdst + kTcOperand;
            if (lane == 0) mbar_arrive_expect_tx(kv_full + 8 * st, __popc(loaded) * 4 * (kBlockSize * 128));
            __syncwarp();
            if (load) {
                const int row = id * kBlockSize;
                const uint32_t off = lane * kBlockSize * 128;
                tma_load_3d(kdst + off, &tmK, 0, kvh, row, kv_full + 8 * st);
                tma_load_3d(kdst + kTcChunk + off, &tmK, 64, kvh, row, kv_full + 8 * st);
                tma_load_3d(vdst + off, &tmV, 0, kvh, row, kv_full + 8 * st);
                tma_load_3d(vdst + kTcChunk + off, &tmV, 64, kvh, row, kv_full + 8 * st);
            }
            // V rows with no token: whole blocks not loaded, and the slots past the context
            // in the sequence's last block (once it has landed)
            for (int b = 0; b < 8; ++b) {
                if ((loaded >> b) & 1u) continue;
                for (int i = lane; i < kBlockSize * 16; i += 32) {
                    const int r = b * kBlockSize + (i >> 4), c = i & 15;
                    const uint32_t a = vdst + (c >> 3) * kTcChunk + r * 128 + ((c & 7) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0) : "memory");
                }
            }
            const int jt = (ctx % kBlockSize) ? nblk_seq - 1 : -1;
            const int bt = jt - j * 8;
            if (bt >= 0 && bt < 8 && ((loaded >> bt) & 1u)) {
                bool landed = true;
                if (lane == 0) landed = mbar_wait_bounded(kv_full + 8 * st, round & 1);
                if (!__shfl_sync(0xffffffffu, landed, 0)) {
                    if (lane == 0) {
                        count_error(p.err);
                        atomicExch(&abort_sh, 1);
                    }
                    break;
                }
                const int r0 = ctx % kBlockSize;
                for (int i = lane; i < (kBlockSize - r0) * 16; i += 32) {
                    const int r = bt * kBlockSize + r0 + (i >> 4), c = i & 15;
                    const uint32_t a = vdst + (c >> 3) * kTcChunk + r * 128 + ((c & 7) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0) : "memory");
                }
            }
            fence_proxy_async_smem();  // these generic stores are read by the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(v_ready + 8 * st);
        }
    } else if (warp == 5) {
        // ================= MMA issuer =================
        const uint32_t idesc_s = instr_desc_bf16(kTcRows, kTcKeys, false);
        const uint32_t idesc_o = instr_desc_bf16(kTcRows, kTcD, true);
        bool alive = true;
        if (lane == 0) alive = mbar_wait_bounded(q_full, 0);
        auto issue_s = [&](int j) -> bool {
            const int st = j % kTcStages, round = j / kTcStages;
            if (!mbar_wait_bounded(kv_full + 8 * st, round & 1)) return false;
            tc_fence_after();
            const uint32_t kb = base + kTcKV + st * 2 * kTcOperand;
            const uint32_t d = tmem + (j & 1) * kTcKeys;
#pragma unroll
            for (int ks = 0; ks < kTcD / 16; ++ks) {
                const uint32_t off = (ks >> 2) * kTcChunk + (ks & 3) * 32;
                umma_ss(d, smem_desc(base + kTcQ + off, 16, 1024), smem_desc(kb + off, 16, 1024), idesc_s, ks > 0);
            }
            umma_commit(s_full + 8 * (j & 1));
            return true;
        };
        if (lane == 0 && alive) alive = issue_s(0);
        for (int j = 0; j < ntiles; ++j) {
            alive = __shfl_sync(0xffffffffu, alive, 0) && !*abort_flag;
            if (!alive) break;
            if (lane == 0) {
                if (j + 1 < ntiles) alive = issue_s(j + 1);
                // P_j written (and O rescaled) by the softmax warps; V's empty rows zeroed
                const int st = j % kTcStages;
                if (alive) alive = mbar_wait_bounded(p_full, j & 1);
                if (alive) alive = mbar_wait_bounded(v_ready + 8 * st, (j / kTcStages) & 1);
                if (alive) {
                    tc_fence_after();
                    const uint32_t vb = base + kTcKV + st * 2 * kTcOperand + kTcOperand;
#pragma unroll
                    for (int ks = 0; ks < kTcKeys / 16; ++ks) {
                        const uint64_t a = smem_desc(base + kTcP + (ks >> 2) * kTcChunk + (ks & 3) * 32, 16, 1024);
                        const uint64_t b = smem_desc(vb + ks * 16 * 128, kTcChunk, 1024);
                        umma_ss(tmem + 256, a, b, idesc_o, j > 0 || ks > 0);
                    }
                    umma_commit(pv_done);
                    umma_commit(kv_empty + 8 * st);
                }
            }
        }
        if (!__shfl_sync(0xffffffffu, alive, 0)) {
            if (lane == 0) {
                count_error(p.err);
                atomicExch(&abort_sh, 1);
            }
        }
    } else {
        // ================= softmax (warps 0-3): thread = query row =================
        const int r = threadIdx.x;                 // 0..127 = TMEM lane
        const int qpos = pos0 + row0 + r;          // this row's position (rows past nq: unused)
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
        float m_ref = -INFINITY, l = 0.f;
        bool alive = true;
        for (int j = 0; j < ntiles; ++j) {
            if (!alive || *abort_flag) break;
            // blocks of this tile that hold tokens (in the table, id in range)
            unsigned okmask = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                const int jb = j * 8 + b;
                const int id = jb < nblk_seq ? __ldg(tab + jb) : -1;
                if (id >= 0 && id < p.num_blocks) okmask |= 1u << b;
            }
            bool w1 = mbar_wait_bounded(s_full + 8 * (j & 1), (j >> 1) & 1);
            if (!__all_sync(0xffffffffu, w1)) {
                alive = false;
                break;
            }
            tc_fence_after();
            // scores of keys j*128 + c, masked: causal, block id out of range
            float x[kTcKeys];
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                float v[32];
                tmem_ld32(lane_addr + (j & 1) * kTcKeys + 32 * c4, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) x[32 * c4 + i] = v[i];
            }
            tmem_wait_ld();
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < kTcKeys; ++c) {
                const int kpos = j * kTcKeys + c;
                const bool valid = kpos <= qpos && ((okmask >> (c >> 4)) & 1u);
                x[c] = valid ? x[c] * p.score_scale : -INFINITY;
                mx = fmaxf(mx, x[c]);
            }
            // the reference max moves only when a score exceeds it by more than 2^8
            float alpha = 1.f;
            const bool move = mx > m_ref + kRescaleThreshold || m_ref == -INFINITY;
            const float m_new = move ? mx : m_ref;
            if (move && m_ref != -INFINITY) alpha = fast_exp2(m_ref - m_new);
            const float mu = m_new == -INFINITY ? 0.f : m_new;
            float sum = 0.f;
            // PV_{j-1} must be done before P is overwritten and before O is read
            if (j > 0) {
                bool w2 = mbar_wait_bounded(pv_done, (j - 1) & 1);
                if (!__all_sync(0xffffffffu, w2)) {
                    alive = false;
                    break;
                }
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
                    for (int c4 = 0; c4 < 4; ++c4) {
                        float v[32];
                        tmem_ld32(lane_addr + 256 + 32 * c4, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] *= alpha;
                        tmem_st32(lane_addr + 256 + 32 * c4, v);
                    }
                    tmem_wait_st();
                }
            }
            l *= alpha;
            m_ref = m_new;
            // P row r as bf16 into the K-major 128-byte-swizzled operand: keys 64c..64c+63 in
            // column chunk c, 16-byte piece q of the row at ((q ^ (r & 7)) << 4)
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float p0 = fast_exp2(x[64 * c + 8 * q + 2 * e] - mu);
                        const float p1 = fast_exp2(x[64 * c + 8 * q + 2 * e + 1] - mu);
                        sum += p0 + p1;
                        w[e] = pack_bf16x2(p0, p1);
                    }
                    const uint32_t a = base + kTcP + c * kTcChunk + r * 128 + ((q ^ (r & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(w[0]), "r"(w[1]),
                                 "r"(w[2]), "r"(w[3])
                                 : "memory");
                }
            l += sum;
            fence_proxy_async_smem();  // generic-proxy P stores -> read by the tensor core
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        if (!alive && lane == 0) {
            count_error(p.err);
            atomicExch(&abort_sh, 1);
        }
        // epilogue: wait for the last PV, normalise and store the row
        if (alive && !*abort_flag) {
            bool w3 = mbar_wait_bounded(pv_done, (ntiles - 1) & 1);
            if (__all_sync(0xffffffffu, w3)) {
                tc_fence_after();
                const float inv = l > 0.f ? 1.f / l : 0.f;
                const bool store = row0 + r < nq;
                __nv_bfloat16* out = p.out + ((size_t)(qs0 + row0 + r) * p.num_heads + h) * kTcD;
#pragma unroll 1
                for (int c4 = 0; c4 < 4; ++c4) {
                    float v[32];
                    tmem_ld32(lane_addr + 256 + 32 * c4, v);
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
    if (warp == 5) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

cudaError_t launch_prefill_tc(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                              const PrefillParams& p, int max_query_len, cudaStream_t stream) {
    const int smem = kTcSmem + 1024;
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int tiles = (max_query_len + kTcRows - 1) / kTcRows;
    return launch_pdl(prefill_tc_kernel, dim3(tiles, p.num_seqs, p.num_heads), dim3(192), smem, stream, tmQ, tmK,
                      tmV, p);
}

}  // namespace pkv
