// Step a3 in FP4 on the 5th-generation tensor cores: lightning-indexer scores from MXFP4
// query heads and keys ("DeepSeek-V4 深度分析报告" Figure 2, "Lightning Indexer FP4
// Precision", and section 3.4: MXFP4 on the QK path of CSA, the indexer scores quantised
// from FP32 to BF16 for the top-k selector).
//
// MXFP4: e2m1 elements, two per byte (element 2j in the low nibble), one UE8M0 scale per
// 32 consecutive elements.  s_i = sum_h w_h * ReLU(q_h . k_i), the heads accumulated by
// fmaf in ascending order in fp32; with select_bf16 each score is then rounded to BF16
// (nearest, ties to even) before it is stored and selected.
//
// A key row is 64 bytes of elements + 4 scale bytes, half the FP8 row: decode stays
// HBM-bound.  The kernel has the FP8 indexer's structure (same work items, persistent CTAs);
// what differs:
//   warp 0 lane 0  TMA producer: per query the heads (H_I x 64 bytes, B operand); per stage
//                  a group of up to three 128-row key tiles (64-byte rows, 64-byte swizzle),
//                  8 x 24 KB in flight;
//   warp 1         TMEM allocation; lane 0 copies the scale factors into TMEM (tcgen05.cp,
//                  32x128b broadcast to the four lane quarters) and issues
//                  tcgen05.mma kind::mxf4.block_scale (M = 128 entries, N = H_I heads,
//                  2 x K = 64 per tile) into one of two sets of three accumulators;
//   warp 2         scale-factor staging: the keys' UE8M0 bytes copied by 4-byte cp.async
//                  straight into the tensor cores' scale layout (row r = r0 + 32 r1: bytes
//                  at 16 r0 + 4 r1 + block), three groups ahead; the heads' scales and the
//                  head weights per query / item;
//   warps 3-14     epilogue in three groups of four, group j taking tile j of every stage
//                  group: tcgen05.ld of one entry row per thread (in halves of 32 heads),
//                  the fmaf chain, the optional BF16 rounding, the score store and the
//                  group maxima.
// Every wait is bounded; a timeout aborts the CTA, drains its own copies and MMAs, frees
// TMEM and reports CSA_DEV_TIMEOUT.
#include "indexer_items.cuh"
#include "launchers.cuh"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kGroupTiles = 3;           // tiles per pipeline stage
constexpr int kStages = 8;               // 8 x 24 KB of key tiles in flight per SM
constexpr int kAccSets = 2;
constexpr int kAux = 3;                  // prefetched items (head weights)
constexpr int kDI = 128;                 // indexer dim (elements)
constexpr int kRowBytes = kDI / 2;       // packed key / head row
constexpr int kTileBytes = kTileRows * kRowBytes;
constexpr int kGroupBytes = kGroupTiles * kTileBytes;
constexpr int kSfBytes = 512;            // scale factors of 128 rows x 4 blocks
constexpr int kFirstEpiWarp = 3;
constexpr int kEpiGroups = kGroupTiles;  // epilogue warp groups: one per tile of a group
constexpr int kEpiWarps = 4 * kEpiGroups;
constexpr int kThreads = 32 * (kFirstEpiWarp + kEpiWarps);

struct Fp4Args {
    const uint8_t* qsf;      // [Q, HI, 4]
    const float* w;          // [Q, HI]
    const uint8_t* ksf;      // [ent_rows, 4]
    const int64_t* seq_len;
    EntryRows er;
    const int32_t* q_seq;
    const int32_t* q_pos;
    float* scores;
    int64_t ld;
    int64_t ent_rows;
    int32_t* st;
    int Q, B, m, max_n;
    int qtiles;
    int chunks_per_q;
    int bf16;                // round each score to BF16 before storing / selecting
    int keys_once;           // no more queries than sequences (decode): each key row is read once
    uint32_t* gmax;          // nullable: group maxima, as in the FP8 indexer
    int64_t ld_g;
};

// TMEM: accumulators (kAccSets x kGroupTiles x HI columns), then the keys' scale columns
// (4 per accumulator), then two sets of 4 scale columns for the heads.
template <int HI>
__host__ __device__ constexpr int acc_cols() { return kAccSets * kGroupTiles * HI; }
template <int HI>
__host__ __device__ constexpr int sfa_col0() { return acc_cols<HI>(); }
template <int HI>
__host__ __device__ constexpr int sfb_col0() { return acc_cols<HI>() + kAccSets * kGroupTiles * 4; }
template <int HI>
__host__ __device__ constexpr uint32_t tmem_cols() {
    constexpr int c = sfb_col0<HI>() + 2 * 4;
    return c <= 32 ? 32u : c <= 64 ? 64u : c <= 128 ? 128u : c <= 256 ? 256u : 512u;
}

// Rearranges the scale bytes of 128 rows (row r's 4 bytes at src + 4 r, rows >= nrows
// taken as 0) into the tensor cores' layout at dst: the 16 bytes at 16 r0 hold rows r0,
// r0 + 32, r0 + 64, r0 + 96.  One warp; lane = r0.
__device__ __forceinline__ void stage_scales(uint8_t* dst, const uint8_t* src, int nrows,
                                             int lane) {
    uint32_t v[4];
#pragma unroll
    for (int r1 = 0; r1 < 4; r1++) {
        const int r = lane + 32 * r1;
        v[r1] = r < nrows ? __ldg(reinterpret_cast<const uint32_t*>(src) + r) : 0u;
    }
    *reinterpret_cast<uint4*>(dst + 16 * lane) = make_uint4(v[0], v[1], v[2], v[3]);
}

// Walks the CTA's groups of tiles in order (items with tiles, kGroupTiles per group).
struct GroupCursor {
    int ii;
    Item x;
    int g0;
    bool valid;
    template <class A>
    __device__ __forceinline__ void seek(const A& a, const Item* items, int64_t v0, int64_t v1,
                                         int n_my) {
        for (; ii < n_my; ii++)
            if (fetch_item(a, items, v0, v1, ii, x, false)) {
                valid = true;
                return;
            }
        valid = false;
    }
    template <class A>
    __device__ __forceinline__ void start(const A& a, const Item* items, int64_t v0, int64_t v1,
                                          int n_my) {
        ii = 0;
        g0 = 0;
        seek(a, items, v0, v1, n_my);
    }
    template <class A>
    __device__ __forceinline__ void next(const A& a, const Item* items, int64_t v0, int64_t v1,
                                         int n_my) {
        g0 += kGroupTiles;
        if (g0 < x.ntiles) return;
        g0 = 0;
        ii++;
        seek(a, items, v0, v1, n_my);
    }
};

// 4-byte asynchronous global -> shared copy; src_bytes = 0 writes zeros without reading.
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// PAGED: the key rows come through the block table (a separate instantiation, so the
// contiguous kernel carries no block-table code).
template <int HI, bool PAGED>
__global__ void __launch_bounds__(kThreads, 1)
    indexer_fp4_kernel(const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_q, const Fp4Args a) {
    using namespace sm100;
    constexpr int kQBytes = HI * kRowBytes;
    // the heads' scale layout is filled for 128 rows (rows >= HI are zero)
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* sA = smem;                                   // [kStages][kGroupTiles][128 x 64]
    uint8_t* sB = sA + kStages * kGroupBytes;             // [2][HI x 64]
    uint8_t* sSfa = sB + 2 * kQBytes;                     // [kStages][kGroupTiles][512]
    uint8_t* sSfb = sSfa + kStages * kGroupTiles * kSfBytes;   // [2][512]
    float* aux = reinterpret_cast<float*>(sSfb + 2 * kSfBytes);  // [kAux][HI]
    uint64_t* bars = reinterpret_cast<uint64_t*>(aux + kAux * HI);
    uint64_t* full = bars;                                // [kStages] key tiles landed
    uint64_t* empty = full + kStages;                     // [kStages] tiles and scales used
    uint64_t* sfafull = empty + kStages;                  // [kStages] key scales staged
    uint64_t* bfull = sfafull + kStages;                  // [2]
    uint64_t* bempty = bfull + 2;                         // [2]
    uint64_t* sfbfull = bempty + 2;                       // [2]
    uint64_t* sfbempty = sfbfull + 2;                     // [2]
    uint64_t* accfull = sfbempty + 2;                     // [kAccSets]
    uint64_t* accempty = accfull + kAccSets;              // [kAccSets]
    uint64_t* auxfull = accempty + kAccSets;              // [kAux]
    uint64_t* auxempty = auxfull + kAux;                  // [kAux]
    uint64_t* drain = auxempty + kAux;                    // [1]
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_smem + 1);
    Item* items = reinterpret_cast<Item*>(tmem_base_smem + 4);   // [kMaxItems]
    int64_t v0, v1;
    cta_range(a, blockIdx.x, gridDim.x, v0, v1);
    const int n_my = v1 > v0 ? (int)(chunk_of(a, v1 - 1) - chunk_of(a, v0) + 1) : 0;

    // As the FP8 indexer: inputs only are read before the score stores, which wait for
    // the previous grid.
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sfafull[s], 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(&bfull[i], 1);
            mbar_init(&bempty[i], 1);
            mbar_init(&sfbfull[i], 1);
            mbar_init(&sfbempty[i], 1);
        }
        for (int i = 0; i < kAccSets; i++) {
            mbar_init(&accfull[i], 1);
            mbar_init(&accempty[i], kEpiWarps);
        }
        for (int i = 0; i < kAux; i++) {
            mbar_init(&auxfull[i], 1);
            mbar_init(&auxempty[i], kEpiWarps);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        mbar_fence_init();
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_q);
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_smem, tmem_cols<HI>());
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_smem;
    if (warp > 0) {
        for (int i = threadIdx.x - 32; i < min(n_my, kMaxItems); i += kThreads - 32) {
            Item x;
            if (!get_item(a, v0, v1, i, x, true)) x.ntiles = 0;
            items[i] = x;
        }
        asm volatile("bar.sync 1, %0;" ::"r"(kThreads - 32) : "memory");
    }

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            int stage = 0;
            uint32_t ephase = 0;
            int nq = 0, cur_q = -1, ng = 0;
            bool ok = true;
            // key rows read once (decode) take the evict-first policy: the key tiles
            // leave L2 first, and the score rows and group maxima the top-k reads next stay
            const uint64_t pol = l2_policy(a.keys_once != 0);
            for (int ii = 0; ii < n_my && ok; ii++) {
                Item x;
                if (!get_item(a, v0, v1, ii, x, false)) continue;
                if (x.q != cur_q) {
                    const int bb = nq & 1;
                    if (!mbar_wait(&bempty[bb], ((nq >> 1) & 1) ^ 1, abort_flag, a.st)) break;
                    mbar_arrive_expect_tx(&bfull[bb], kQBytes);
                    tma_load_2d(sB + bb * kQBytes, &tmap_q, &bfull[bb], 0, x.q * HI);
                    nq++;
                    cur_q = x.q;
                }
                for (int g0 = 0; g0 < x.ntiles; g0 += kGroupTiles) {
                    const int gt = min(kGroupTiles, x.ntiles - g0);
                    if (!mbar_wait(&empty[stage], ephase ^ 1, abort_flag, a.st)) {
                        ok = false;
                        break;
                    }
                    if constexpr (!PAGED) {
                        mbar_arrive_expect_tx(&full[stage], gt * kTileBytes);
                        for (int j = 0; j < gt; j++)
                            tma_load_2d_hint(sA + stage * kGroupBytes + j * kTileBytes, &tmap_k,
                                             &full[stage], 0,
                                             (int32_t)(x.row0 + (int64_t)(x.tile0 + g0 + j) * kTileRows),
                                             pol);
                    } else {
                        int32_t rows[kGroupTiles][kTilePages];
                        int nb = 0;
                        for (int j = 0; j < gt; j++) nb += tile_pages(a, x, x.tile0 + g0 + j, rows[j]);
                        mbar_arrive_expect_tx(&full[stage], (uint32_t)nb * (kPageRows * kRowBytes));
                        for (int j = 0; j < gt; j++)
#pragma unroll
                            for (int p = 0; p < kTilePages; p++)
                                if (rows[j][p] >= 0)
                                    tma_load_2d_hint(sA + stage * kGroupBytes + j * kTileBytes +
                                                         p * (kPageRows * kRowBytes),
                                                     &tmap_k, &full[stage], 0, rows[j][p], pol);
                    }
                    ng++;
                    if (++stage == kStages) {
                        stage = 0;
                        ephase ^= 1;
                    }
                }
            }
            for (int s = 0; s < kStages; s++) {
                const int cnt = ng / kStages + (s < ng % kStages ? 1 : 0);
                if (cnt) mbar_drain(&full[s], (cnt - 1) & 1, a.st);
            }
            for (int i = 0; i < 2; i++) {
                const int cnt = (nq - i + 1) / 2;
                if (cnt) mbar_drain(&bfull[i], (cnt - 1) & 1, a.st);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- scale copies and MMA issuer ----------------
            int stage = 0;
            uint32_t sphase = 0;
            int nq = 0, cur_q = -1, ng = 0;
            uint64_t bdesc = 0;
            uint32_t sfb = 0;
            bool ok = true;
            for (int ii = 0; ii < n_my && ok; ii++) {
                Item x;
                if (!fetch_item(a, items, v0, v1, ii, x, false)) continue;
                if (x.q != cur_q) {
                    // the previous query's heads (smem and TMEM scales) are free once the
                    // MMAs issued so far finish
                    if (nq > 0) mma_commit(&bempty[(nq - 1) & 1]);
                    const int bb = nq & 1;
                    if (!mbar_wait(&bfull[bb], (nq >> 1) & 1, abort_flag, a.st) ||
                        !mbar_wait(&sfbfull[bb], (nq >> 1) & 1, abort_flag, a.st))
                        break;
                    tc_fence_after();
                    bdesc = smem_desc_k_sw64(sB + bb * kQBytes);
                    sfb = tmem_base + (uint32_t)(sfb_col0<HI>() + 4 * bb);
                    tmem_cp_32x128b_x4(sfb, smem_desc_rows16(sSfb + bb * kSfBytes));
                    mma_commit(&sfbempty[bb]);
                    nq++;
                    cur_q = x.q;
                }
                for (int g0 = 0; g0 < x.ntiles; g0 += kGroupTiles) {
                    const int gt = min(kGroupTiles, x.ntiles - g0);
                    const int set = ng & (kAccSets - 1);
                    if (!mbar_wait(&accempty[set], ((ng / kAccSets) & 1) ^ 1, abort_flag, a.st) ||
                        !mbar_wait(&full[stage], sphase, abort_flag, a.st) ||
                        !mbar_wait(&sfafull[stage], sphase, abort_flag, a.st)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t adesc = smem_desc_k_sw64(sA + stage * kGroupBytes);
                    const uint32_t d0 = tmem_base + (uint32_t)(set * kGroupTiles * HI);
                    const uint32_t sfa0 = tmem_base + (uint32_t)(sfa_col0<HI>() + set * kGroupTiles * 4);
#pragma unroll
                    for (int j = 0; j < kGroupTiles; j++)
                        if (j < gt)
                            tmem_cp_32x128b_x4(sfa0 + 4 * j,
                                               smem_desc_rows16(sSfa + (stage * kGroupTiles + j) * kSfBytes));
#pragma unroll
                    for (int kk = 0; kk < kDI / 64; kk++) {   // K = 64 e2m1 = 32 bytes per MMA
                        const uint32_t idesc = instr_desc_mxf4(kTileRows, HI, 2 * kk, 2 * kk);
                        const uint32_t sel = (uint32_t)(2 * kk) << 30;
#pragma unroll
                        for (int j = 0; j < kGroupTiles; j++)
                            if (j < gt)
                                mma_mxf4(d0 + (uint32_t)(j * HI),
                                         adesc + (uint64_t)((j * kTileBytes) >> 4) + 2 * kk,
                                         bdesc + 2 * kk, idesc, (sfa0 + 4 * j) | sel, sfb | sel,
                                         kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&empty[stage]);
                    mma_commit(&accfull[set]);
                    ng++;
                    if (++stage == kStages) {
                        stage = 0;
                        sphase ^= 1;
                    }
                }
            }
            mma_commit(drain);
            mbar_drain(drain, 0, a.st);
        }
    } else if (warp == 2) {
        // ---------------- scale staging and head weights ----------------
        // The keys' scale bytes go straight to their places in the tensor cores' layout by
        // 4-byte asynchronous copies, kLookAhead groups ahead of the group whose scales are
        // being released to the MMA thread, so that no global-load latency is serialised
        // per group.  The heads' scales and weights are loaded when the released group is
        // the first of its query / item.
        constexpr int kLookAhead = 3;
        GroupCursor iss, rel;
        iss.start(a, items, v0, v1, n_my);
        rel.start(a, items, v0, v1, n_my);
        int istage = 0, rstage = 0;
        uint32_t iphase = 0;
        int issued = 0, released = 0;
        int nq = 0, cur_q = -1, nit = 0, cur_ii = -1;
        bool ok = true;
        while (rel.valid && ok) {
            while (iss.valid && issued - released < kLookAhead) {
                if (!mbar_wait_warp(&empty[istage], iphase ^ 1, abort_flag, a.st)) {
                    ok = false;
                    break;
                }
                const int gt = min(kGroupTiles, iss.x.ntiles - iss.g0);
                for (int j = 0; j < gt; j++) {
                    const int64_t e0 = (int64_t)(iss.x.tile0 + iss.g0 + j) * kTileRows;
                    const uint32_t dst = smem_addr(sSfa + (istage * kGroupTiles + j) * kSfBytes) + 16 * lane;
                    if constexpr (!PAGED) {
#pragma unroll
                        for (int r1 = 0; r1 < 4; r1++) {
                            const int64_t row = iss.x.row0 + e0 + lane + 32 * r1;
                            const bool in = row < a.ent_rows;
                            cp_async4(dst + 4 * r1, a.ksf + (in ? row : 0) * 4, in ? 4u : 0u);
                        }
                    } else {
                        int64_t rows[4];
#pragma unroll
                        for (int r1 = 0; r1 < 4; r1++) {
                            const int64_t e = e0 + lane + 32 * r1;
                            rows[r1] = e < iss.x.n_vis ? a.er.row(iss.x.b, e) : -1;
                        }
#pragma unroll
                        for (int r1 = 0; r1 < 4; r1++) {
                            const bool in = rows[r1] >= 0 && rows[r1] < a.ent_rows;
                            cp_async4(dst + 4 * r1, a.ksf + (in ? rows[r1] : 0) * 4, in ? 4u : 0u);
                        }
                    }
                }
                cp_async_commit();
                issued++;
                if (++istage == kStages) {
                    istage = 0;
                    iphase ^= 1;
                }
                iss.next(a, items, v0, v1, n_my);
            }
            if (!ok) break;
            if (rel.ii != cur_ii) {
                // the released group is the first of its item
                cur_ii = rel.ii;
                if (rel.x.q != cur_q) {
                    const int bb = nq & 1;
                    if (!mbar_wait_warp(&sfbempty[bb], ((nq >> 1) & 1) ^ 1, abort_flag, a.st)) break;
                    stage_scales(sSfb + bb * kSfBytes, a.qsf + (int64_t)rel.x.q * HI * 4, HI, lane);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sfbfull[bb]);
                    nq++;
                    cur_q = rel.x.q;
                }
                const int slot = nit % kAux;
                if (!mbar_wait_warp(&auxempty[slot], ((nit / kAux) & 1) ^ 1, abort_flag, a.st)) break;
#pragma unroll
                for (int h = lane; h < HI; h += 32)
                    aux[slot * HI + h] = __ldg(a.w + (int64_t)rel.x.q * HI + h);
                __syncwarp();
                if (lane == 0) mbar_arrive(&auxfull[slot]);
                nit++;
            }
            // the released group's copies are done once at most (issued - released - 1)
            // later groups are pending
            const int pending = issued - released - 1;
            if (pending >= 2) {
                cp_async_wait<2>();
            } else if (pending == 1) {
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sfafull[rstage]);
            released++;
            if (++rstage == kStages) rstage = 0;
            rel.next(a, items, v0, v1, n_my);
        }
        // no copy of this warp may still be writing shared memory when the CTA ends
        cp_async_wait<0>();
    } else {
        // ---------------- epilogue (warps 3..14) ----------------
        const int grp = (warp - kFirstEpiWarp) / 4;
        const int quarter = warp & 3;
        const int row_in_tile = quarter * 32 + lane;
        int ng = 0, nit = 0;
        bool ok = true;
        bool waited = false;
        for (int ii = 0; ii < n_my && ok; ii++) {
            Item x;
            if (!fetch_item(a, items, v0, v1, ii, x, false)) continue;
            const int slot = nit % kAux;
            if (!mbar_wait_warp(&auxfull[slot], (nit / kAux) & 1, abort_flag, a.st)) break;
            float ws[HI];
#pragma unroll
            for (int h = 0; h < HI; h += 4) {
                const float4 v4 = *reinterpret_cast<const float4*>(aux + slot * HI + h);
                ws[h] = v4.x;
                ws[h + 1] = v4.y;
                ws[h + 2] = v4.z;
                ws[h + 3] = v4.w;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&auxempty[slot]);
            nit++;
            float* srow = a.scores + (int64_t)x.q * a.ld;
            for (int g0 = 0; g0 < x.ntiles; g0 += kGroupTiles) {
                const int gt = min(kGroupTiles, x.ntiles - g0);
                const int set = ng & (kAccSets - 1);
                if (!mbar_wait_warp(&accfull[set], (ng / kAccSets) & 1, abort_flag, a.st)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (!waited) {
                    pdl_wait();
                    waited = true;
                }
                // epilogue group grp takes tile grp of the group; the accumulator row is
                // read in halves of at most 32 heads (fewer live registers), the heads still
                // accumulated in ascending order
                const int j = grp;
                if (j < gt) {
                    const int tt = g0 + j;
                    const int e = (x.tile0 + tt) * kTileRows + row_in_tile;
                    const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) +
                                           (uint32_t)((set * kGroupTiles + j) * HI);
                    constexpr int kHalf = HI < 32 ? HI : 32;
                    float acc = 0.f;
#pragma unroll
                    for (int h0 = 0; h0 < HI; h0 += kHalf) {
                        uint32_t d[kHalf];
                        if constexpr (kHalf == 32) {
                            tmem_ld32(taddr + (uint32_t)h0, d);
                        } else {
                            tmem_ld16(taddr + (uint32_t)h0, d);
                        }
                        tmem_ld_wait();
#pragma unroll
                        for (int h = 0; h < kHalf; h++)
                            acc = fmaf(ws[h0 + h], fmaxf(__uint_as_float(d[h]), 0.f), acc);
                    }
                    uint32_t key = 0u;
                    if (e < x.n_vis) {
                        if (a.bf16) acc = __bfloat162float(__float2bfloat16_rn(acc));
                        if (acc != acc) flag(a.st, CSA_DEV_NAN);
                        srow[e] = acc;
                        key = order_key(acc);
                    }
                    if (a.gmax) {
                        key = __reduce_max_sync(0xffffffffu, key);
                        const int e0 = e - lane;
                        if (lane == 0 && e0 < x.n_vis) a.gmax[(int64_t)x.q * a.ld_g + (e0 >> 5)] = key;
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&accempty[set]);
                ng++;
            }
        }
    }

    pdl_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tmem_cols<HI>());
    }
}

template <int HI>
size_t smem_bytes() {
    return 1024 + kStages * kGroupBytes + 2 * HI * kRowBytes +
           kStages * kGroupTiles * kSfBytes + 2 * kSfBytes + kAux * HI * sizeof(float) +
           (3 * kStages + 8 + 2 * kAccSets + 2 * kAux + 1) * 8 + 16 + kMaxItems * sizeof(Item);
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
    static EncodeFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(p);
        tried = true;
    }
    return fn;
}

// Row-major [rows x 64] byte matrix, boxes of box_rows x 64 bytes, 64-byte swizzle.
bool make_rows64_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
    EncodeFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)kRowBytes, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kRowBytes};
    const cuuint32_t box[2] = {(cuuint32_t)kRowBytes, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

int sm_count_fp4() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

template <int HI>
cudaError_t launch_hi(const uint8_t* qI, const uint8_t* kI, const Fp4Args& args,
                      cudaStream_t stream) {
    CUtensorMap mk, mq;
    if (!make_rows64_map(&mk, kI, (uint64_t)args.ent_rows, args.er.bt ? kPageRows : kTileRows) ||
        !make_rows64_map(&mq, qI, (uint64_t)args.Q * HI, HI))
        return cudaErrorInvalidValue;
    const size_t sm = smem_bytes<HI>();
    auto kernel = args.er.bt ? indexer_fp4_kernel<HI, true> : indexer_fp4_kernel<HI, false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sm);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (int64_t)args.Q * args.qtiles;
    const int grid = (int)(tiles < (int64_t)sm_count_fp4() ? tiles : (int64_t)sm_count_fp4());
    LaunchScope scope(kKIndexerFp4, stream);
    return launch_pdl(kernel, dim3(grid), dim3(kThreads), sm, stream, mk, mq,
                      args);
}

}  // namespace

bool indexer_fp4_supported(int HI, int dI) {
    return dI == kDI && (HI == 16 || HI == 32 || HI == 64);
}

cudaError_t launch_indexer_fp4(const uint8_t* qI, const uint8_t* qI_sf, const float* w,
                               const uint8_t* kI, const uint8_t* kI_sf, int64_t ent_rows,
                               const int64_t* seq_len, const EntryRows& er,
                               const int32_t* q_seq, const int32_t* q_pos, int Q, int B, int HI,
                               int m, int max_n, int bf16, float* scores, int64_t ld,
                               int32_t* st, cudaStream_t stream, uint32_t* gmax, int64_t ld_g) {
    if (Q == 0 || max_n == 0 || ent_rows == 0) return cudaSuccess;
    Fp4Args args;
    args.qsf = qI_sf;
    args.w = w;
    args.ksf = kI_sf;
    args.seq_len = seq_len;
    args.er = er;
    args.q_seq = q_seq;
    args.q_pos = q_pos;
    args.scores = scores;
    args.ld = ld;
    args.ent_rows = ent_rows;
    args.st = st;
    args.Q = Q;
    args.B = B;
    args.m = m;
    args.max_n = max_n;
    args.keys_once = Q <= B;
    args.bf16 = bf16;
    args.gmax = gmax;
    args.ld_g = ld_g;
    args.qtiles = (max_n + kTileRows - 1) / kTileRows;
    args.chunks_per_q = (args.qtiles + kChunkTiles - 1) / kChunkTiles;
    switch (HI) {
        case 64: return launch_hi<64>(qI, kI, args, stream);
        case 32: return launch_hi<32>(qI, kI, args, stream);
        case 16: return launch_hi<16>(qI, kI, args, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace csa
