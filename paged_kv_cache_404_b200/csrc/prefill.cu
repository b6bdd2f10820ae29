// prefill.cu -- causal multi-token paged attention (the prompt pass), bf16.
//
// What it computes: sequence s has nq new query tokens, the last nq of its
// context_len tokens, whose K/V the caller has already written into the pool
// (a prompt is allocated first and its last block then filled; attention reads
// the blocks through the table in logical order: iplexlaw.co.kr, section on
// logical vs physical order).  Query i sits at position p = context_len - nq + i
// and attends to every token t <= p (gyaansetu.com, what the KV cache holds):
//   out[i][h] = softmax_t(scale * q[i][h] . K[t][g]) V[t][g],  g = h / (Hq/Hkv).
// A whole prompt (nq = context_len), a prompt after a cached prefix and a
// chunk of a long prompt are the same call.
//
// Work decomposition.  A CTA takes 16*CW query rows of one sequence and one
// query head, and streams that sequence's K/V blocks 0 .. (last row's
// position)/16 through a ring of STAGES shared-memory stages: one producer warp
// walks the block table and issues TMA loads (the same 3-D tensor maps as the
// decode: [slots][kv heads][head_dim], 16-slot x 1-head x 128-byte boxes,
// 128-byte swizzle) onto per-stage "full" mbarriers; CW consumer warps each own
// 16 query rows, FlashAttention-2 style: S = Q K^T on tensor cores
// (mma.m16n8k16, Q in registers, K by ldmatrix), online softmax in base 2 with
// the causal mask, P re-used in registers as the A operand of O += P V (V by
// ldmatrix.trans), then arrive on the stage's "empty" mbarrier.  Tiles are
// launched last-rows-first (the longest rows first).
#include "pkv_common.cuh"

namespace pkv {


constexpr int kPfD = 128;
constexpr int kPfTile = kBlockSize * kPfD * 2;  // one block of one head, K or V: 16 rows x 256 B
constexpr int kPfStage = 2 * kPfTile;           // K tile + V tile

template <int CW, int STAGES>
__global__ void __launch_bounds__((CW + 1) * 32, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const PrefillParams p) {
    constexpr int ROWS = 16 * CW;
    extern __shared__ uint8_t smem_raw[];
    // full[st] at 8*st, empty[st] at 8*(STAGES+st), tail_ready at 8*(2*STAGES)
    __shared__ __align__(8) uint64_t bars[2 * STAGES + 1];
    __shared__ int stage_ok[STAGES];
    const uint32_t ring = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t bar0 = smem_u32(&bars[0]);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;

    if (threadIdx.x == 0) {
        for (int st = 0; st < STAGES; ++st) {
            mbar_init(bar0 + 8 * st, 1);
            mbar_init(bar0 + 8 * (STAGES + st), CW);
        }
        mbar_init(bar0 + 8 * (2 * STAGES), 1);
        fence_barrier_init();
    }
    if (warp == CW && lane == 0) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();

    const int s = blockIdx.y, h = blockIdx.z, kvh = h / p.group;
    const int tile = gridDim.x - 1 - blockIdx.x;
    const int qs0 = p.query_start[s];
    const int nq = p.query_start[s + 1] - qs0;
    const int ctx = p.context_lens[s];
    const int row0 = tile * ROWS;
    if (row0 >= nq) return;  // the whole CTA leaves together, before any barrier use
    if (nq > ctx || ctx > p.max_blocks_per_seq * kBlockSize) {
        // inconsistent lengths: zero outputs for these rows, count once per sequence
        if (tile == 0 && h == 0 && threadIdx.x == 0) count_error(p.err);
        const int rows = min(ROWS, nq - row0);
        for (int e = threadIdx.x; e < rows * kPfD; e += blockDim.x) {
            const int r = e / kPfD, d = e - r * kPfD;
            p.out[((size_t)(qs0 + row0 + r) * p.num_heads + h) * kPfD + d] = __float2bfloat16(0.f);
        }
        return;
    }
    const int pos0 = ctx - nq;                       // position of query row 0
    const int last_row = min(row0 + ROWS, nq) - 1;
    const int nblk = (pos0 + last_row) / kBlockSize + 1;
    // blocks this tile covers first (the previous tile stops before them): bad ids counted here
    const int count_from = tile == 0 ? 0 : (pos0 + row0 - 1) / kBlockSize + 1;
    const int32_t* tab = p.block_tables + (size_t)s * p.max_blocks_per_seq;
    // the sequence's last block holds slots past the context when ctx % 16 != 0;
    // if this CTA reads it, the producer zeroes those V rows once it has landed
    const int j_tail = (ctx % kBlockSize) && (ctx - 1) / kBlockSize < nblk ? (ctx - 1) / kBlockSize : -1;
    const uint32_t tail_ready = bar0 + 8 * (2 * STAGES);

    if (warp == CW) {
        // ---- producer: block ids 32 at a time, TMA loads into the ring
        for (int j0 = 0; j0 < nblk; j0 += 32) {
            const int id_l = j0 + lane < nblk ? __ldg(tab + j0 + lane) : -1;
            const int jn = min(32, nblk - j0);
            for (int jj = 0; jj < jn; ++jj) {
                const int id = __shfl_sync(0xffffffffu, id_l, jj);
                const int j = j0 + jj;
                bool alive = true;
                if (lane == 0) {
                    const int st = j % STAGES, round = j / STAGES;
                    if (round > 0 && !mbar_wait_bounded(bar0 + 8 * (STAGES + st), (round - 1) & 1)) {
                        count_error(p.err);
                        alive = false;
                    } else {
                        const bool ok = id >= 0 && id < p.num_blocks;
                        if (!ok && h == 0 && j >= count_from) count_error(p.err);
                        stage_ok[st] = ok;
                        const uint32_t full = bar0 + 8 * st;
                        const uint32_t dk = ring + st * kPfStage, dv = dk + kPfTile;
                        const int row = (ok ? id : 0) * kBlockSize;
                        mbar_arrive_expect_tx(full, kPfStage);
                        tma_load_3d(dk, &tmK, 0, kvh, row, full);
                        tma_load_3d(dk + kBlockSize * 128, &tmK, 64, kvh, row, full);
                        tma_load_3d(dv, &tmV, 0, kvh, row, full);
                        tma_load_3d(dv + kBlockSize * 128, &tmV, 64, kvh, row, full);
                    }
                }
                if (!__shfl_sync(0xffffffffu, alive, 0)) return;
            }
        }
        if (j_tail >= 0) {
            // rows past the context may hold anything (NaN included): zero them in V
            // so that a zero probability cannot meet them in the PV product
            const int st = j_tail % STAGES;
            bool landed = true;
            if (lane == 0) landed = mbar_wait_bounded(bar0 + 8 * st, (j_tail / STAGES) & 1);
            if (!__shfl_sync(0xffffffffu, landed, 0)) {
                if (lane == 0) count_error(p.err);
                return;
            }
            __syncwarp();  // lane 0's stage_ok store is visible to the warp
            if (stage_ok[st]) {
                const uint32_t vt = ring + st * kPfStage + kPfTile;
                const int nz = (kBlockSize - ctx % kBlockSize) * 16;  // 16-byte chunks
                for (int i = lane; i < nz; i += 32) {
                    const int r = ctx % kBlockSize + (i >> 4), c = i & 15;
                    const uint32_t a = vt + (c >> 3) * (kBlockSize * 128) + r * 128 + (c & 7) * 16;
                    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0) : "memory");
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(tail_ready);
        }
        return;
    }

    // ---- consumers: 16 query rows each
    const int wrow0 = row0 + 16 * warp;
    const int qp_lo = pos0 + wrow0 + g, qp_hi = qp_lo + 8;  // positions of this thread's two rows
    const bool has_rows = wrow0 <= last_row;
    const int wblk = has_rows ? (pos0 + min(wrow0 + 15, last_row)) / kBlockSize + 1 : 0;

    // Q as A fragments: rows g / g+8, columns 2t.. of each 16-wide k step
    uint32_t qf[kPfD / 16][4];
    {
        const bool v_lo = wrow0 + g < nq, v_hi = wrow0 + g + 8 < nq;
        const __nv_bfloat16* q_lo = p.q + ((size_t)(qs0 + (v_lo ? wrow0 + g : 0)) * p.num_heads + h) * kPfD;
        const __nv_bfloat16* q_hi = p.q + ((size_t)(qs0 + (v_hi ? wrow0 + g + 8 : 0)) * p.num_heads + h) * kPfD;
#pragma unroll
        for (int ks = 0; ks < kPfD / 16; ++ks) {
            const int d0 = ks * 16 + 2 * t;
            qf[ks][0] = v_lo ? *reinterpret_cast<const uint32_t*>(q_lo + d0) : 0u;
            qf[ks][1] = v_hi ? *reinterpret_cast<const uint32_t*>(q_hi + d0) : 0u;
            qf[ks][2] = v_lo ? *reinterpret_cast<const uint32_t*>(q_lo + d0 + 8) : 0u;
            qf[ks][3] = v_hi ? *reinterpret_cast<const uint32_t*>(q_hi + d0 + 8) : 0u;
        }
    }
    // swizzled lane offsets in a tile: chunk c of row r at r*128 + ((c ^ (r & 7)) << 4),
    // the two 64-element halves of a row 2048 bytes apart
    //  koff[j]: K as the B operand, matrices (tok 0-7, c 2j) (0-7, 2j+1) (8-15, 2j) (8-15, 2j+1)
    //  voff[j]: V as the B operand (.trans), matrices (tok 0-7, c 2j) (8-15, 2j) (0-7, 2j+1) (8-15, 2j+1)
    uint32_t koff[4], voff[4];
    {
        const int ktok = (lane & 7) + ((lane >> 4) & 1) * 8, kc = (lane >> 3) & 1;
        const int vtok = (lane & 7) + ((lane >> 3) & 1) * 8, vc = lane >> 4;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            koff[j] = ktok * 128 + ((((2 * j + kc) & 7) ^ (ktok & 7)) << 4);
            voff[j] = vtok * 128 + ((((2 * j + vc) & 7) ^ (vtok & 7)) << 4);
        }
    }

    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
    float o[kPfD / 8][4];
#pragma unroll
    for (int n = 0; n < kPfD / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

    for (int j = 0; j < nblk; ++j) {
        const int st = j % STAGES, round = j / STAGES;
        const uint32_t kt = ring + st * kPfStage, vt = kt + kPfTile;
        if (!mbar_wait_bounded(bar0 + 8 * st, round & 1)) {
            if (lane == 0) count_error(p.err);
            return;
        }
        if (j == j_tail && !mbar_wait_bounded(tail_ready, 0)) {
            if (lane == 0) count_error(p.err);
            return;
        }
        const bool ok = stage_ok[st] != 0;
        if (ok && j < wblk) {
            float sc[2][4];
#pragma unroll
            for (int n = 0; n < 2; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < kPfD / 16; ++ks) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(kt + (ks >> 2) * (kBlockSize * 128) + koff[ks & 3], b0, b1, b2, b3);
                mma_bf16(sc[0], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b0, b1);
                mma_bf16(sc[1], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b2, b3);
            }
            // causal mask and base-2 scores; this thread's keys: j*16 + 8n + 2t + {0, 1}
            float x[2][4];
            float bm_lo = -INFINITY, bm_hi = -INFINITY;
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int kpos = j * kBlockSize + 8 * n + 2 * t + (e & 1);
                    const int qp = e < 2 ? qp_lo : qp_hi;
                    x[n][e] = kpos <= qp ? sc[n][e] * p.score_scale : -INFINITY;
                }
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                bm_lo = fmaxf(bm_lo, fmaxf(x[n][0], x[n][1]));
                bm_hi = fmaxf(bm_hi, fmaxf(x[n][2], x[n][3]));
            }
#pragma unroll
            for (int off = 1; off < 4; off <<= 1) {
                bm_lo = fmaxf(bm_lo, __shfl_xor_sync(0xffffffffu, bm_lo, off));
                bm_hi = fmaxf(bm_hi, __shfl_xor_sync(0xffffffffu, bm_hi, off));
            }
            const float mn_lo = fmaxf(m_lo, bm_lo), mn_hi = fmaxf(m_hi, bm_hi);
            const float mu_lo = mn_lo == -INFINITY ? 0.f : mn_lo, mu_hi = mn_hi == -INFINITY ? 0.f : mn_hi;
            const float al_lo = fast_exp2(m_lo - mu_lo), al_hi = fast_exp2(m_hi - mu_hi);
            float pr[2][4];
            float s_lo = 0.f, s_hi = 0.f;
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                pr[n][0] = fast_exp2(x[n][0] - mu_lo);
                pr[n][1] = fast_exp2(x[n][1] - mu_lo);
                pr[n][2] = fast_exp2(x[n][2] - mu_hi);
                pr[n][3] = fast_exp2(x[n][3] - mu_hi);
                s_lo += pr[n][0] + pr[n][1];
                s_hi += pr[n][2] + pr[n][3];
            }
            l_lo = l_lo * al_lo + s_lo;
            l_hi = l_hi * al_hi + s_hi;
            m_lo = mn_lo;
            m_hi = mn_hi;
            if (__any_sync(0xffffffffu, al_lo != 1.f || al_hi != 1.f)) {
#pragma unroll
                for (int n = 0; n < kPfD / 8; ++n) {
                    o[n][0] *= al_lo;
                    o[n][1] *= al_lo;
                    o[n][2] *= al_hi;
                    o[n][3] *= al_hi;
                }
            }
            // P (16 rows x 16 keys) as the A operand of the PV product
            const uint32_t a0 = pack_bf16x2(pr[0][0], pr[0][1]), a1 = pack_bf16x2(pr[0][2], pr[0][3]);
            const uint32_t a2 = pack_bf16x2(pr[1][0], pr[1][1]), a3 = pack_bf16x2(pr[1][2], pr[1][3]);
#pragma unroll
            for (int jj = 0; jj < kPfD / 16; ++jj) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(vt + (jj >> 2) * (kBlockSize * 128) + voff[jj & 3], b0, b1, b2, b3);
                mma_bf16(o[2 * jj], a0, a1, a2, a3, b0, b1);
                mma_bf16(o[2 * jj + 1], a0, a1, a2, a3, b2, b3);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar0 + 8 * (STAGES + st));
    }

    // ---- epilogue: full row sums, normalise, store rows < nq
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
        l_lo += __shfl_xor_sync(0xffffffffu, l_lo, off);
        l_hi += __shfl_xor_sync(0xffffffffu, l_hi, off);
    }
    const float inv_lo = l_lo > 0.f ? 1.f / l_lo : 0.f, inv_hi = l_hi > 0.f ? 1.f / l_hi : 0.f;
    const int r_lo = wrow0 + g, r_hi = r_lo + 8;
    if (r_lo < nq) {
        __nv_bfloat16* out = p.out + ((size_t)(qs0 + r_lo) * p.num_heads + h) * kPfD + 2 * t;
#pragma unroll
        for (int n = 0; n < kPfD / 8; ++n)
            *reinterpret_cast<uint32_t*>(out + 8 * n) = pack_bf16x2(o[n][0] * inv_lo, o[n][1] * inv_lo);
    }
    if (r_hi < nq) {
        __nv_bfloat16* out = p.out + ((size_t)(qs0 + r_hi) * p.num_heads + h) * kPfD + 2 * t;
#pragma unroll
        for (int n = 0; n < kPfD / 8; ++n)
            *reinterpret_cast<uint32_t*>(out + 8 * n) = pack_bf16x2(o[n][2] * inv_hi, o[n][3] * inv_hi);
    }
}

#ifndef PKV_PF_WARPS
#define PKV_PF_WARPS 4
#endif
#ifndef PKV_PF_STAGES
#define PKV_PF_STAGES 4
#endif

cudaError_t launch_prefill(const CUtensorMap& tmK, const CUtensorMap& tmV, const PrefillParams& p, int max_query_len,
                           cudaStream_t stream) {
    constexpr int CW = PKV_PF_WARPS, ST = PKV_PF_STAGES;
    const int smem = ST * kPfStage + 1024;
    auto kern = prefill_kernel<CW, ST>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int tiles = (max_query_len + 16 * CW - 1) / (16 * CW);
    return launch_pdl(kern, dim3(tiles, p.num_seqs, p.num_heads), dim3((CW + 1) * 32), smem, stream, tmK, tmV, p);
}

}  // namespace pkv
