// decode_tc.cu -- paged decode attention, BF16 / FP8 caches, tensor cores.
//
// What it computes (PagedAttention): for one new query token per sequence,
// out[s][h] = softmax(scale * q[s][h] . K[t]) over t < len_s, applied to V[t],
// where token t of sequence s is read through its block table at row
// (table[s][t / 16], t % 16) of the pool (glossary entry "PagedAttention",
// "Como funciona la paginacion" and its worked example).  The attention is
// tiled FlashAttention-style -- one 16-token block at a time with a running
// max and sum, so no score matrix is written to memory (same page, "Tecnicas
// relacionadas") -- and query heads that share a key/value head (grouped-query
// attention, same section) are served by a single read of each K/V tile.
//
// Work decomposition.  A unit is (sequence, partition, kv head).  The kernel
// is persistent: one CTA per SM, each warp an independent worker that takes
// units from an atomic counter in the plan's longest-first order.  Each warp
// owns a ring of STAGES shared-memory stages; a stage holds the K tile and the
// V tile of one block for its kv head (16 rows of head_dim elements each),
// fetched by TMA (3-D tensor map over [slots][kv heads][head_dim], 128-byte
// swizzle, box = 16 slots x 1 head x 128 bytes) and completing on per-stage
// mbarriers.  Lane 0 issues the loads STAGES blocks ahead of the block the
// warp is computing.
//
// Per block, in "swap-AB" form so the 16 tokens are the M=16 side of
// mma.m16n8k16 and the (up to 8) query heads of the group are N=8:
//   S^T[16 tok x 8 heads]  = K_tile[16 x D] * Q^T[D x 8]      (D/16 MMAs)
//   online softmax over the tokens of each head column (base-2 exponent)
//   O^T[D x 8 heads]      += V_tile^T[D x 16] * P^T[16 x 8]   (D/16 MMAs)
// P^T's B fragment is the transpose of S^T's accumulator fragment, produced
// with movmatrix.  BF16 tiles feed ldmatrix(.trans); FP8 tiles are converted to
// f16 in registers (exact) and use f16 MMAs, with the per-tensor scales folded
// into the score scale and the output.
#include "pkv_common.cuh"

namespace pkv {


template <bool FP8, int D>
struct TileCfg {
    static constexpr int kElem = FP8 ? 1 : 2;
    static constexpr int kRowBytes = D * kElem;            // bytes of one token row of one head
    static constexpr int kSub = kRowBytes / 128;            // 128-byte swizzle atoms per row
    static constexpr int kBoxElems = 128 / kElem;           // TMA box inner extent (elements)
    static constexpr int kTileBytes = kBlockSize * kRowBytes;
    static constexpr int kStageBytes = 2 * kTileBytes;      // K tile + V tile
    static_assert(kRowBytes % 128 == 0, "rows must be whole 128-byte swizzle atoms");
};

template <bool FP8, int D, int NT, int WARPS, int STAGES, int BPS, bool GROUPED>
__global__ void __launch_bounds__(WARPS * 32, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const DecodeParams p) {
    using C = TileCfg<FP8, D>;
    constexpr int KS = D / 16;  // k-steps of the score MMA == m-tiles of the output MMA
    static_assert(STAGES >= 2 && STAGES < 64, "ring depth");
    static_assert(BPS >= 1 && BPS <= STAGES, "blocks per step fit in the ring");

    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[WARPS][2 * STAGES];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t ring = base + warp * STAGES * C::kStageBytes;
    const uint32_t bar0 = smem_u32(&bars[warp][0]);  // K barrier of stage st at bar0 + 8*st, V at + 8*(STAGES+st)

    if (lane == 0) {
        if (warp == 0) {
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
        }
        for (int st = 0; st < 2 * STAGES; ++st) mbar_init(bar0 + 8 * st, 1);
        fence_barrier_init();
    }
    __syncwarp();
    // everything above overlaps the plan kernel; its outputs are read below
    pdl_wait();
    pdl_trigger();

    // Lane-dependent byte offsets inside a swizzled tile (chunk c of row r sits
    // at r*128 + ((c ^ (r & 7)) << 4) within its 16-row x 128-byte atom), computed
    // once; per block only the stage base is added.  Atoms of the tile (64-element
    // halves of a bf16 D=128 row) add 2048 bytes each.
    //  koff[j]: ldmatrix of K, matrices (rows 0-7 | 8-15) x (chunk 2j | 2j+1)
    //  voff[j]: ldmatrix.trans of V, matrices (rows 0-7, 2j) (0-7, 2j+1) (8-15, 2j) (8-15, 2j+1)
    //  foff[j][r]: FP8 V words at rows 2t (+r) of chunk 2j + (g >> 2), byte 4 (g & 3)
    uint32_t koff[4], voff[4], foff[4][2];
    {
        const int krow = (lane & 7) + ((lane >> 3) & 1) * 8, kh = lane >> 4;
        const int vrow = (lane & 7) + (lane >> 4) * 8, vh = (lane >> 3) & 1;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            koff[j] = krow * 128 + ((((2 * j + kh) & 7) ^ (krow & 7)) << 4);
            voff[j] = vrow * 128 + ((((2 * j + vh) & 7) ^ (vrow & 7)) << 4);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int row = 2 * t + r;
                foff[j][r] = row * 128 + ((((2 * j + (g >> 2)) & 7) ^ (row & 7)) << 4) + (g & 3) * 4;
            }
        }
    }

    const int num_units = p.hdr->num_units;
    const int G = p.group;
    uint32_t seqno = 0;  // blocks this warp has consumed so far (stage = seqno % STAGES)

    for (;;) {
        int u = 0;
        if (lane == 0) u = atomicAdd(&p.hdr->counter, 1);
        u = __shfl_sync(0xffffffffu, u, 0);
        if (u >= num_units) break;
        const int4 item = p.items[u / p.num_kv_heads];
        const int kvh = u - (u / p.num_kv_heads) * p.num_kv_heads;
        int s_item = item.x;
        const int part = item.y;
        // A subgroup item (shared-prefix decode) serves M sequences that hold the
        // same physical blocks: one read of each K/V tile, M*G score columns
        // (member i's query heads are columns i*G .. i*G+G-1).  The claim that
        // they hold the same blocks came from the caller: it is checked here for
        // this item's blocks, and if any member's table differs the item runs
        // once per member (M passes of one member each), as if ungrouped.
        int M_item = 1, mbase_item = 0, npass = 1;
        if constexpr (GROUPED) {
            if (s_item < 0) {
                const int4 si = p.sub_info[-s_item - 1];
                mbase_item = si.x;
                M_item = si.y;
                s_item = p.sub_members[mbase_item];
                const int32_t* t_first = p.block_tables + (size_t)s_item * p.max_blocks_per_seq + item.z;
                bool same = true;
                for (int j = lane; j < item.w; j += 32) {
                    const int r = __ldg(t_first + j);
#pragma unroll 4
                    for (int mi = 1; mi < M_item; ++mi) {
                        const int sm = p.sub_members[mbase_item + mi];
                        same = (__ldg(p.block_tables + (size_t)sm * p.max_blocks_per_seq + item.z + j) == r) & same;
                    }
                }
                if (!__all_sync(0xffffffffu, same)) npass = M_item;
            }
        }
        for (int pass = 0; pass < npass; ++pass) {
        const int M = npass > 1 ? 1 : M_item;
        const int mbase = mbase_item + (npass > 1 ? pass : 0);
        const int s = pass > 0 ? p.sub_members[mbase] : s_item;
        const int ncols = M * G;
        const int nt_act = GROUPED ? (ncols + 7) >> 3 : NT;  // n-tiles holding a column
        const int L = clamped_len(p, s, false);
        const int blk0 = item.z;
        const int t0 = blk0 * kBlockSize;
        const int t1 = min(L, t0 + item.w * kBlockSize);
        const int nblk = (t1 - t0 + kBlockSize - 1) / kBlockSize;
        const int32_t* tab = p.block_tables + (size_t)s * p.max_blocks_per_seq + blk0;

        // Block ids, 32 at a time: lane i holds block (32*chunk + i); the next
        // chunk is loaded one chunk ahead of use.
        auto load_ids = [&](int chunk) -> int {
            const int j = chunk * 32 + lane;
            return j < nblk ? __ldg(tab + j) : -1;
        };
        int ids_cur = load_ids(0);
        int ids_nxt = load_ids(1);
        int chunk_cur = 0;
        unsigned long long okmask = 0;  // bit (j & 63): block j's id was in range

        // Q^T fragments (B operand): n = query head of the group, k = head_dim,
        // and the score scale of this thread's two score columns (heads 2t, 2t+1).
        // FP8 cache: the products run in f16, where every E4M3 code is exact, but
        // f16 does not span bf16's range.  So each head's q is first multiplied
        // by a power of two 2^e that brings its largest magnitude into
        // [2^14, 2^15): exact, no entry can overflow, and every entry down to
        // 2^-28 of that maximum keeps all of its bf16 bits in f16.  The head's
        // score column then takes 2^-e along with the score scale.
        uint32_t qf[NT][KS][2];
        float cs[NT][2];
        const int hq0 = kvh * G;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            int hh = nt * 8 + g, sq = s;
            bool hv = hh < G;
            if constexpr (GROUPED) {
                const int c = hh;
                hv = c < ncols;
                const int mi = hv ? c / G : 0;
                hh = c - mi * G;
                if (mi > 0) sq = p.sub_members[mbase + mi];
            }
            const __nv_bfloat16* qrow =
                static_cast<const __nv_bfloat16*>(p.q) + ((size_t)sq * p.num_heads + hq0 + (hv ? hh : 0)) * D;
            if constexpr (!FP8) {
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    const int d0 = ks * 16 + 2 * t;
                    qf[nt][ks][0] = hv ? *reinterpret_cast<const uint32_t*>(qrow + d0) : 0u;
                    qf[nt][ks][1] = hv ? *reinterpret_cast<const uint32_t*>(qrow + d0 + 8) : 0u;
                }
                cs[nt][0] = cs[nt][1] = p.score_scale;
            } else {
                // k positions {2t, 2t+1, 2t+8, 2t+9} of step ks hold head_dim 16ks+4t+{0,1,2,3};
                // the four lanes t = 0..3 of group g hold the whole row of head g
                uint2 w[KS];
                uint32_t amax_bits = 0;
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    w[ks] = hv ? *reinterpret_cast<const uint2*>(qrow + ks * 16 + 4 * t) : make_uint2(0u, 0u);
                    // |x| of a bf16 orders like its bits with the sign cleared
                    amax_bits = max(amax_bits, max(max(w[ks].x & 0x7FFFu, (w[ks].x >> 16) & 0x7FFFu),
                                                   max(w[ks].y & 0x7FFFu, (w[ks].y >> 16) & 0x7FFFu)));
                }
                amax_bits = max(amax_bits, __shfl_xor_sync(0xffffffffu, amax_bits, 1));
                amax_bits = max(amax_bits, __shfl_xor_sync(0xffffffffu, amax_bits, 2));
                // e = 14 - floor(log2 max|q|), kept in [-126, 126] so that 2^e and
                // 2^-e are normal floats (a bf16 subnormal maximum then still lands
                // at or above 2^-7); an all-zero head keeps e = 0
                const int ex = amax_bits != 0 ? (int)(amax_bits >> 7) - 127 : 14;
                const int e = min(max(14 - ex, -126), 126);
                const float up = __uint_as_float((uint32_t)(127 + e) << 23);
                const float down = __uint_as_float((uint32_t)(127 - e) << 23) * p.score_scale;
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    qf[nt][ks][0] = pack_f16x2(__uint_as_float(w[ks].x << 16) * up,
                                               __uint_as_float(w[ks].x & 0xFFFF0000u) * up);
                    qf[nt][ks][1] = pack_f16x2(__uint_as_float(w[ks].y << 16) * up,
                                               __uint_as_float(w[ks].y & 0xFFFF0000u) * up);
                }
                // score column c is head c of this n-tile, held by lanes 4c .. 4c+3
                cs[nt][0] = __shfl_sync(0xffffffffu, down, 8 * t);
                cs[nt][1] = __shfl_sync(0xffffffffu, down, 8 * t + 4);
            }
        }

        // Issue the TMA loads of block j of this unit into its stage (all lanes
        // call it: the block id is broadcast with a shuffle).
        auto issue = [&](int j) {
            const int ch = j >> 5;
            if (ch != chunk_cur) {
                ids_cur = ids_nxt;
                ids_nxt = load_ids(ch + 1);
                chunk_cur = ch;
            }
            const int id = __shfl_sync(0xffffffffu, ids_cur, j & 31);
            const bool ok = id >= 0 && id < p.num_blocks;
            if (ok) okmask |= 1ull << (j & 63);
            else okmask &= ~(1ull << (j & 63));
            if (lane == 0) {
                if (!ok && kvh == 0) count_error(p.err);
                const uint32_t st = (seqno + j) % STAGES;
                const uint32_t bk = bar0 + 8 * st, bv = bar0 + 8 * (STAGES + st);
                const uint32_t dk = ring + st * C::kStageBytes, dv = dk + C::kTileBytes;
                const int row = (ok ? id : 0) * kBlockSize;
                mbar_arrive_expect_tx(bk, C::kTileBytes);
#pragma unroll
                for (int sub = 0; sub < C::kSub; ++sub)
                    tma_load_3d(dk + sub * (kBlockSize * 128), &tmK, sub * C::kBoxElems, kvh, row, bk);
                mbar_arrive_expect_tx(bv, C::kTileBytes);
#pragma unroll
                for (int sub = 0; sub < C::kSub; ++sub)
                    tma_load_3d(dv + sub * (kBlockSize * 128), &tmV, sub * C::kBoxElems, kvh, row, bv);
            }
        };

        const int npro = nblk < STAGES ? nblk : STAGES;
        for (int j = 0; j < npro; ++j) issue(j);
        int issued = npro;

        float m[NT][2], l[NT][2], oacc[NT][KS][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            m[nt][0] = m[nt][1] = -INFINITY;
            l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
            for (int i = 0; i < KS; ++i) oacc[nt][i][0] = oacc[nt][i][1] = oacc[nt][i][2] = oacc[nt][i][3] = 0.f;
        }

        // ---- per-tile pieces ------------------------------------------------
        // S^T[16 tok x 8 heads] of the K tile at `kt` (even and odd k-steps in two
        // independent accumulation chains, summed at the end)
        auto scores = [&](uint32_t kt, float (&sc)[NT][4]) {
            float sc2[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) sc[nt][e] = sc2[nt][e] = 0.f;
            if constexpr (!FP8) {
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    uint32_t a0, a1, a2, a3;
                    ldmatrix_x4(kt + (ks >> 2) * (kBlockSize * 128) + koff[ks & 3], a0, a1, a2, a3);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        if (nt < nt_act)
                            mma_bf16((ks & 1) ? sc2[nt] : sc[nt], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
                }
            } else {
#pragma unroll
                for (int kp = 0; kp < KS / 2; ++kp) {
                    uint32_t r0, r1, r2, r3;
                    ldmatrix_x4(kt + koff[kp], r0, r1, r2, r3);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if (nt >= nt_act) continue;
                        mma_f16(sc[nt], e4m3x2_to_f16x2(r0), e4m3x2_to_f16x2(r1), e4m3x2_to_f16x2(r0 >> 16),
                                e4m3x2_to_f16x2(r1 >> 16), qf[nt][2 * kp][0], qf[nt][2 * kp][1]);
                        mma_f16(sc2[nt], e4m3x2_to_f16x2(r2), e4m3x2_to_f16x2(r3), e4m3x2_to_f16x2(r2 >> 16),
                                e4m3x2_to_f16x2(r3 >> 16), qf[nt][2 * kp + 1][0], qf[nt][2 * kp + 1][1]);
                    }
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) sc[nt][e] += sc2[nt][e];
        };

        // O^T[D x 8] += V^T[D x 16] P^T[16 x 8] for the V tile at `vt`
        auto accumulate_pv = [&](uint32_t vt, const uint32_t (&pb0)[NT], const uint32_t (&pb1)[NT]) {
            if constexpr (!FP8) {
#pragma unroll
                for (int i = 0; i < KS; ++i) {
                    uint32_t a0, a1, a2, a3;
                    ldmatrix_x4_trans(vt + (i >> 2) * (kBlockSize * 128) + voff[i & 3], a0, a1, a2, a3);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        if (nt < nt_act) mma_bf16(oacc[nt][i], a0, a1, a2, a3, pb0[nt], pb1[nt]);
                }
            } else {
#pragma unroll
                for (int q4 = 0; q4 < D / 32; ++q4) {
                    // bytes 32*q4 + 4g .. +3 of token rows 2t, 2t+1, 2t+8, 2t+9 (rows r and
                    // r+8 share a swizzle phase: +8 rows = +1024 bytes)
                    const uint32_t w0 = lds32(vt + foff[q4][0]);
                    const uint32_t w1 = lds32(vt + foff[q4][1]);
                    const uint32_t w2 = lds32(vt + foff[q4][0] + 8 * 128);
                    const uint32_t w3 = lds32(vt + foff[q4][1] + 8 * 128);
                    // pair up the two tokens of each k-pair: (tok a, tok b) per head_dim column
                    const uint32_t x01lo = __byte_perm(w0, w1, 0x5140), x01hi = __byte_perm(w0, w1, 0x7362);
                    const uint32_t x23lo = __byte_perm(w2, w3, 0x5140), x23hi = __byte_perm(w2, w3, 0x7362);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if (nt >= nt_act) continue;
                        // m-tile 2*q4: rows g -> column 32q4+4g, g+8 -> 32q4+4g+1
                        mma_f16(oacc[nt][2 * q4], e4m3x2_to_f16x2(x01lo), e4m3x2_to_f16x2(x01lo >> 16),
                                e4m3x2_to_f16x2(x23lo), e4m3x2_to_f16x2(x23lo >> 16), pb0[nt], pb1[nt]);
                        // m-tile 2*q4+1: rows g -> column 32q4+4g+2, g+8 -> 32q4+4g+3
                        mma_f16(oacc[nt][2 * q4 + 1], e4m3x2_to_f16x2(x01hi), e4m3x2_to_f16x2(x01hi >> 16),
                                e4m3x2_to_f16x2(x23hi), e4m3x2_to_f16x2(x23hi >> 16), pb0[nt], pb1[nt]);
                    }
                }
            }
        };

        // ---- main loop: BPS blocks per step (one softmax reduction per step) ----
        bool dead = false;
        int j = 0;
        for (; j < nblk; j += BPS) {
            const int nb = min(BPS, nblk - j);  // warp-uniform
            uint32_t stb[BPS], parb[BPS], kt[BPS], vt[BPS];
            bool okb[BPS];
            int nvalid[BPS];
            bool any_ok = false;
#pragma unroll
            for (int b = 0; b < BPS; ++b) {
                const int jb = j + b;
                stb[b] = (seqno + jb) % STAGES;
                parb[b] = ((seqno + jb) / STAGES) & 1u;
                kt[b] = ring + stb[b] * C::kStageBytes;
                vt[b] = kt[b] + C::kTileBytes;
                okb[b] = b < nb && ((okmask >> (jb & 63)) & 1ull);
                nvalid[b] = b < nb ? min(kBlockSize, t1 - (t0 + jb * kBlockSize)) : 0;
                any_ok = any_ok || okb[b];
            }

            bool waited = true;
#pragma unroll
            for (int b = 0; b < BPS; ++b)
                if (b < nb) waited = waited && mbar_wait_bounded(bar0 + 8 * stb[b], parb[b]);
            if (!__all_sync(0xffffffffu, waited)) {
                dead = true;
                break;
            }
            float sc[BPS][NT][4];
#pragma unroll
            for (int b = 0; b < BPS; ++b)
                if (okb[b]) scores(kt[b], sc[b]);

#pragma unroll
            for (int b = 0; b < BPS; ++b)
                if (b < nb) waited = waited && mbar_wait_bounded(bar0 + 8 * (STAGES + stb[b]), parb[b]);
            if (!__all_sync(0xffffffffu, waited)) {
                dead = true;
                break;
            }

            if (any_ok) {
                // ---- online softmax over the step's tokens (rows g and g+8 of each block)
                uint32_t pb0[BPS][NT], pb1[BPS][NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (nt >= nt_act) {
#pragma unroll
                        for (int b = 0; b < BPS; ++b) pb0[b][nt] = pb1[b][nt] = 0u;
                        continue;
                    }
                    float x[BPS][4];
                    float b0 = -INFINITY, b1 = -INFINITY;
#pragma unroll
                    for (int b = 0; b < BPS; ++b) {
                        const bool vlo = okb[b] && g < nvalid[b], vhi = okb[b] && g + 8 < nvalid[b];
                        x[b][0] = vlo ? sc[b][nt][0] * cs[nt][0] : -INFINITY;
                        x[b][1] = vlo ? sc[b][nt][1] * cs[nt][1] : -INFINITY;
                        x[b][2] = vhi ? sc[b][nt][2] * cs[nt][0] : -INFINITY;
                        x[b][3] = vhi ? sc[b][nt][3] * cs[nt][1] : -INFINITY;
                        b0 = fmaxf(b0, fmaxf(x[b][0], x[b][2]));
                        b1 = fmaxf(b1, fmaxf(x[b][1], x[b][3]));
                    }
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) {
                        b0 = fmaxf(b0, __shfl_xor_sync(0xffffffffu, b0, o));
                        b1 = fmaxf(b1, __shfl_xor_sync(0xffffffffu, b1, o));
                    }
                    const float mn0 = fmaxf(m[nt][0], b0), mn1 = fmaxf(m[nt][1], b1);
                    const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
                    const float al0 = fast_exp2(m[nt][0] - mu0), al1 = fast_exp2(m[nt][1] - mu1);
                    float s0 = 0.f, s1 = 0.f;
#pragma unroll
                    for (int b = 0; b < BPS; ++b) {
                        const float p0 = fast_exp2(x[b][0] - mu0), p2 = fast_exp2(x[b][2] - mu0);
                        const float p1 = fast_exp2(x[b][1] - mu1), p3 = fast_exp2(x[b][3] - mu1);
                        s0 += p0 + p2;
                        s1 += p1 + p3;
                        // accumulator fragment rows = tokens, cols = heads; transpose into
                        // the B fragment of P^T (rows = tokens as k, cols = heads as n)
                        if constexpr (!FP8) {
                            pb0[b][nt] = movmatrix_trans(pack_bf16x2(p0, p1));
                            pb1[b][nt] = movmatrix_trans(pack_bf16x2(p2, p3));
                        } else {
                            pb0[b][nt] = movmatrix_trans(pack_f16x2(p0, p1));
                            pb1[b][nt] = movmatrix_trans(pack_f16x2(p2, p3));
                        }
                    }
                    l[nt][0] = l[nt][0] * al0 + s0;
                    l[nt][1] = l[nt][1] * al1 + s1;
                    m[nt][0] = mn0;
                    m[nt][1] = mn1;
                    // rescale the accumulator only if some running max moved (rare
                    // after the first blocks); the test is warp-uniform
                    if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
                        for (int i = 0; i < KS; ++i) {
                            oacc[nt][i][0] *= al0;
                            oacc[nt][i][1] *= al1;
                            oacc[nt][i][2] *= al0;
                            oacc[nt][i][3] *= al1;
                        }
                    }
                }

                // Rows past the context hold stale data (possibly NaN): zero them so
                // that a zero probability cannot meet a NaN in the MMA.
                bool zeroed = false;
#pragma unroll
                for (int b = 0; b < BPS; ++b) {
                    if (okb[b] && nvalid[b] < kBlockSize) {
                        const int per_row = C::kSub * 8;
                        const int nz = (kBlockSize - nvalid[b]) * per_row;
                        for (int i = lane; i < nz; i += 32) {
                            const int r = nvalid[b] + i / per_row, c = i - (i / per_row) * per_row;
                            const uint32_t a = vt[b] + (c >> 3) * (kBlockSize * 128) + r * 128 + (c & 7) * 16;
                            asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0) : "memory");
                        }
                        zeroed = true;
                    }
                }
                if (zeroed) {
                    fence_proxy_async_smem();
                    __syncwarp();
                }

#pragma unroll
                for (int b = 0; b < BPS; ++b)
                    if (okb[b]) accumulate_pv(vt[b], pb0[b], pb1[b]);
            }
            __syncwarp();
#pragma unroll
            for (int b = 0; b < BPS; ++b)
                if (b < nb && issued < nblk) {
                    issue(issued);
                    ++issued;
                }
        }

        if (dead) {
            // A load never completed: wait (bounded) for the other loads still in
            // flight into this warp's ring, report, and stop this warp.
            for (int k = j; k < issued; ++k) {
                const uint32_t st = (seqno + k) % STAGES;
                const uint32_t par = ((seqno + k) / STAGES) & 1u;
                mbar_wait_bounded(bar0 + 8 * st, par, 1LL << 28);
                mbar_wait_bounded(bar0 + 8 * (STAGES + st), par, 1LL << 28);
            }
            if (lane == 0) {
                atomicExch(&p.hdr->timeout, 1);
                count_error(p.err);
            }
            return;
        }
        seqno += nblk;

        // ---- epilogue: full l per head column, then out or the partition's (m, l, o)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                if (nt >= nt_act) continue;
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) l[nt][c] += __shfl_xor_sync(0xffffffffu, l[nt][c], o);
            }
        bool split = p.nparts[s] > 1;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                int hh = nt * 8 + 2 * t + c, so = s;
                if constexpr (GROUPED) {
                    const int col = hh;
                    if (col >= ncols) continue;
                    const int mi = col / G;
                    hh = col - mi * G;
                    if (mi > 0) {
                        so = p.sub_members[mbase + mi];
                        split = p.nparts[so] > 1;
                    } else {
                        split = p.nparts[s] > 1;
                    }
                } else {
                    if (hh >= G) continue;
                }
                const int hq = hq0 + hh;
                const float inv = l[nt][c] > 0.f ? p.out_scale / l[nt][c] : 0.f;
                if (!split) {
                    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + ((size_t)so * p.num_heads + hq) * D;
                    if constexpr (!FP8) {
#pragma unroll
                        for (int i = 0; i < KS; ++i) {
                            o[16 * i + g] = __float2bfloat16(oacc[nt][i][c] * inv);
                            o[16 * i + 8 + g] = __float2bfloat16(oacc[nt][i][c + 2] * inv);
                        }
                    } else {
#pragma unroll
                        for (int q4 = 0; q4 < D / 32; ++q4) {
                            const uint32_t lo = pack_bf16x2(oacc[nt][2 * q4][c] * inv, oacc[nt][2 * q4][c + 2] * inv);
                            const uint32_t hi =
                                pack_bf16x2(oacc[nt][2 * q4 + 1][c] * inv, oacc[nt][2 * q4 + 1][c + 2] * inv);
                            *reinterpret_cast<uint2*>(o + 32 * q4 + 4 * g) = make_uint2(lo, hi);
                        }
                    }
                } else {
                    const size_t slot = ((size_t)so * p.num_heads + hq) * p.max_parts + part;
                    float* o = p.part_o + slot * D;
                    if constexpr (!FP8) {
#pragma unroll
                        for (int i = 0; i < KS; ++i) {
                            o[16 * i + g] = oacc[nt][i][c] * inv;
                            o[16 * i + 8 + g] = oacc[nt][i][c + 2] * inv;
                        }
                    } else {
#pragma unroll
                        for (int q4 = 0; q4 < D / 32; ++q4)
                            *reinterpret_cast<float4*>(o + 32 * q4 + 4 * g) =
                                make_float4(oacc[nt][2 * q4][c] * inv, oacc[nt][2 * q4][c + 2] * inv,
                                            oacc[nt][2 * q4 + 1][c] * inv, oacc[nt][2 * q4 + 1][c + 2] * inv);
                    }
                    if (g == 0) p.part_ml[slot] = make_float2(m[nt][c], l[nt][c]);
                }
            }
        }  // pass
    }
}

template <bool FP8, int D, int NT, int WARPS, int STAGES, int BPS, bool GROUPED = false>
static cudaError_t launch_tc(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecodeParams& p, int num_sms,
                             cudaStream_t stream) {
    using C = TileCfg<FP8, D>;
    const int smem = WARPS * STAGES * C::kStageBytes + 1024;
    auto kern = decode_tc_kernel<FP8, D, NT, WARPS, STAGES, BPS, GROUPED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(num_sms), dim3(WARPS * 32), smem, stream, tmK, tmV, p);
}

// Launch shapes, chosen by measurement on B200: warps per CTA (one CTA per SM),
// ring stages per warp and blocks per main-loop step (one softmax reduction per
// step).  Shared memory per CTA = warps * stages * 2 tiles (+1 KB alignment slack).
struct Shape {
    int warps, stages, bps;
};
constexpr Shape kBf16D128{12, 2, 1};
constexpr Shape kBf16D64{8, 6, 1};
constexpr Shape kFp8{16, 3, 2};
constexpr Shape kGrouped{12, 2, 1};  // shared-prefix variant (bf16, head_dim 128, 16 score columns)

int decode_tc_warps(bool fp8, int head_dim, bool grouped) {
    if (grouped) return kGrouped.warps;
    if (fp8) return kFp8.warps;
    return head_dim == 128 ? kBf16D128.warps : kBf16D64.warps;
}

bool decode_tc_groupable(bool fp8, int head_dim, int group) { return !fp8 && head_dim == 128 && group <= 8; }

cudaError_t launch_decode_tc(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecodeParams& p, bool fp8,
                             int num_sms, cudaStream_t stream) {
    const int nt = (p.group + 7) / 8;
    if (p.num_groups > 0) {
        if (!decode_tc_groupable(fp8, p.head_dim, p.group)) return cudaErrorInvalidValue;
        return launch_tc<false, 128, 2, kGrouped.warps, kGrouped.stages, kGrouped.bps, true>(
            tmK, tmV, p, num_sms, stream);
    }
    if (fp8) {
        if (p.head_dim != 128) return cudaErrorInvalidValue;
        return nt == 1 ? launch_tc<true, 128, 1, kFp8.warps, kFp8.stages, kFp8.bps>(tmK, tmV, p, num_sms, stream)
                       : launch_tc<true, 128, 2, kFp8.warps, kFp8.stages, kFp8.bps>(tmK, tmV, p, num_sms, stream);
    }
    if (p.head_dim == 128)
        return nt == 1
                   ? launch_tc<false, 128, 1, kBf16D128.warps, kBf16D128.stages, kBf16D128.bps>(tmK, tmV, p, num_sms, stream)
                   : launch_tc<false, 128, 2, kBf16D128.warps, kBf16D128.stages, kBf16D128.bps>(tmK, tmV, p, num_sms, stream);
    return nt == 1
               ? launch_tc<false, 64, 1, kBf16D64.warps, kBf16D64.stages, kBf16D64.bps>(tmK, tmV, p, num_sms, stream)
               : launch_tc<false, 64, 2, kBf16D64.warps, kBf16D64.stages, kBf16D64.bps>(tmK, tmV, p, num_sms, stream);
}

}  // namespace pkv
