// Step a3 on the 5th-generation tensor cores: lightning-indexer scores.
//
// "DeepSeek-V4 深度分析报告" 2.1 CSA: the lightning indexer scores every visible
// compressed entry for the query; s_i = ks_i * sum_h (w_h * qs_h) * ReLU(q_h . k_i), the
// heads accumulated by fmaf in ascending order in fp32 (the definition all paths share).
//
// Decode is HBM-bound (each 132-byte key row is read once and feeds 64 x 128 MACs, about
// 124 FLOP/byte), but that intensity still needs the tensor pipe to keep up with HBM.
// Persistent CTAs walk a static list of work items (query, chunk of 8 tiles of 128
// entries); tiles are aligned to the query's sequence, so every entry is always computed
// in the same tile row by the same instructions whatever the batch.  Roles per CTA
// (6 warps):
//   warp 0 lane 0  TMA producer: per item the query's heads (H_I x 128 e4m3, B operand),
//                  per tile 128 key rows (128 x 128 e4m3, A operand), 128-byte swizzle,
//                  into a 4-stage ring;
//   warp 1         TMEM allocation; lane 0 issues tcgen05.mma kind::f8f6f4
//                  (M=128 entries, N=H_I heads, 4 x K=32) into one of two TMEM
//                  accumulators and commits to the stage's and accumulator's barriers;
//   warps 2-5      epilogue: tcgen05.ld of one entry row (all heads) per thread, the
//                  fixed-order fmaf chain, the key scale, a coalesced score store.
// Every wait is bounded; a timeout aborts the CTA, drains its own copies and MMAs,
// frees TMEM and reports CSA_DEV_TIMEOUT.
#include <mutex>

#include "launchers.cuh"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kStages = 4;
constexpr int kTileRows = 128;           // entries per tile (MMA M)
constexpr int kDI = 128;                 // indexer dim (MMA K total, bytes per key row)
constexpr int kTileBytes = kTileRows * kDI;
constexpr int kChunkTiles = 8;           // tiles per work item
constexpr int kThreads = 192;
constexpr int kMaxItems = 512;            // work items per CTA resolved up front

struct IdxArgs {
    const float* qs;
    const float* w;
    const float* ks;
    const int64_t* seq_len;
    const int64_t* ent_off;
    const int32_t* q_seq;
    const int32_t* q_pos;
    float* scores;
    int64_t ld;
    int64_t ent_rows;
    int32_t* st;
    int Q, B, m, max_n, chunks_per_q, total_items;
};

struct Item {
    int q;
    int n_vis;
    int tile0;
    int ntiles;
    int64_t row0;
};

// Decodes work item `it`; false when it has no tiles.  Every role calls this with the same
// arguments and so walks the same item sequence.
__device__ __forceinline__ bool get_item(const IdxArgs& a, int it, Item& x, bool report) {
    x.q = it / a.chunks_per_q;
    const int c = it - x.q * a.chunks_per_q;
    const int b = a.q_seq[x.q];
    const int t = a.q_pos[x.q];
    if (b < 0 || b >= a.B || t < 0 || (int64_t)t >= a.seq_len[b]) {
        if (report && c == 0) flag(a.st, CSA_DEV_OOB);
        return false;
    }
    int n = (t + 1) / a.m;
    if (n > a.max_n) {
        if (report && c == 0) flag(a.st, CSA_DEV_CAPACITY);
        n = a.max_n;
    }
    x.row0 = a.ent_off[b];
    const int64_t avail = a.ent_rows - x.row0;
    if ((int64_t)n > avail) {
        if (report && c == 0) flag(a.st, CSA_DEV_OOB);
        n = avail > 0 ? (int)avail : 0;
    }
    x.n_vis = n;
    x.tile0 = c * kChunkTiles;
    const int tiles = (n + kTileRows - 1) / kTileRows;
    x.ntiles = min(kChunkTiles, tiles - x.tile0);
    return x.ntiles > 0;
}

// Item ii of this CTA: from the table built at kernel start, or decoded directly past it.
__device__ __forceinline__ bool fetch_item(const IdxArgs& a, const Item* items, int ii, Item& x,
                                           bool report) {
    if (ii < kMaxItems) {
        x = items[ii];
        return x.ntiles > 0;
    }
    return get_item(a, blockIdx.x + ii * gridDim.x, x, report);
}

template <int HI>
__global__ void __launch_bounds__(kThreads, 2)
    indexer_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_q, const IdxArgs a) {
    using namespace sm100;
    constexpr int kQBytes = HI * kDI;
    constexpr uint32_t kIdesc = instr_desc(0, 0, kTileRows, HI);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* sA = smem;                                  // [kStages][128 x 128]
    uint8_t* sB = sA + kStages * kTileBytes;             // [2][HI x 128]
    uint64_t* bars = reinterpret_cast<uint64_t*>(sB + 2 * kQBytes);
    uint64_t* full = bars;                               // [kStages]
    uint64_t* empty = full + kStages;                    // [kStages]
    uint64_t* bfull = empty + kStages;                   // [2]
    uint64_t* bempty = bfull + 2;                        // [2]
    uint64_t* accfull = bempty + 2;                      // [2]
    uint64_t* accempty = accfull + 2;                    // [2]
    uint64_t* drain = accempty + 2;                      // [1]
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_smem + 1);
    Item* items = reinterpret_cast<Item*>(tmem_base_smem + 4);   // [kMaxItems]
    // this CTA's work items: it = blockIdx.x + i * gridDim.x
    const int n_my = blockIdx.x < a.total_items
                         ? (a.total_items - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
    // resolve their metadata (dependent loads) in parallel, once; later items on the fly
    for (int i = threadIdx.x; i < min(n_my, kMaxItems); i += kThreads) {
        Item x;
        if (!get_item(a, blockIdx.x + i * gridDim.x, x, true)) x.ntiles = 0;
        items[i] = x;
    }

    // The indexer reads only its inputs (keys and query heads), never an earlier kernel's
    // output, and its score writes are safe once it has started (the previous step's top-k
    // finished before the kernel before this one passed its own wait): let the next kernel
    // launch right away; the wait at the end keeps completion ordered for later kernels.
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(&bfull[i], 1);
            mbar_init(&bempty[i], 1);
            mbar_init(&accfull[i], 1);
            mbar_init(&accempty[i], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        mbar_fence_init();
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_q);
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_smem, 2 * HI < 32 ? 32 : 2 * HI);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_smem;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            int stage = 0;
            uint32_t ephase = 0;
            int nitem = 0;
            int issued[kStages] = {};
            int bissued[2] = {0, 0};
            bool ok = true;
            for (int ii = 0; ii < n_my && ok; ii++) {
                Item x;
                if (!fetch_item(a, items, ii, x, false)) continue;
                const int bb = nitem & 1;
                if (!mbar_wait(&bempty[bb], ((nitem >> 1) & 1) ^ 1, abort_flag, a.st)) break;
                mbar_arrive_expect_tx(&bfull[bb], kQBytes);
                tma_load_2d(sB + bb * kQBytes, &tmap_q, &bfull[bb], 0, x.q * HI);
                bissued[bb]++;
                nitem++;
                for (int tt = 0; tt < x.ntiles; tt++) {
                    if (!mbar_wait(&empty[stage], ephase ^ 1, abort_flag, a.st)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], kTileBytes);
                    tma_load_2d(sA + stage * kTileBytes, &tmap_k, &full[stage], 0,
                                (int32_t)(x.row0 + (int64_t)(x.tile0 + tt) * kTileRows));
                    issued[stage]++;
                    if (++stage == kStages) {
                        stage = 0;
                        ephase ^= 1;
                    }
                }
            }
            // drain: every copy this thread issued must have landed before smem is released
            for (int s = 0; s < kStages; s++)
                if (issued[s]) mbar_drain(&full[s], (issued[s] - 1) & 1, a.st);
            for (int i = 0; i < 2; i++)
                if (bissued[i]) mbar_drain(&bfull[i], (bissued[i] - 1) & 1, a.st);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            int stage = 0;
            uint32_t sphase = 0;
            int nitem = 0, nacc = 0;
            bool ok = true;
            for (int ii = 0; ii < n_my && ok; ii++) {
                Item x;
                if (!fetch_item(a, items, ii, x, false)) continue;
                const int bb = nitem & 1;
                if (!mbar_wait(&bfull[bb], (nitem >> 1) & 1, abort_flag, a.st)) break;
                tc_fence_after();
                const uint64_t bdesc = smem_desc_k_sw128(sB + bb * kQBytes);
                for (int tt = 0; tt < x.ntiles; tt++) {
                    const int ab = nacc & 1;
                    if (!mbar_wait(&accempty[ab], ((nacc >> 1) & 1) ^ 1, abort_flag, a.st) ||
                        !mbar_wait(&full[stage], sphase, abort_flag, a.st)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t adesc = smem_desc_k_sw128(sA + stage * kTileBytes);
                    const uint32_t d = tmem_base + (uint32_t)(ab * HI);
#pragma unroll
                    for (int kk = 0; kk < kDI / 32; kk++)   // K = 32 e4m3 = 32 bytes per MMA
                        mma_f8f6f4(d, adesc + 2 * kk, bdesc + 2 * kk, kIdesc, kk > 0 ? 1u : 0u);
                    mma_commit(&empty[stage]);
                    mma_commit(&accfull[ab]);
                    nacc++;
                    if (++stage == kStages) {
                        stage = 0;
                        sphase ^= 1;
                    }
                }
                if (ok) mma_commit(&bempty[bb]);
                nitem++;
            }
            // drain: all issued MMAs complete before TMEM is released
            mma_commit(drain);
            mbar_drain(drain, 0, a.st);
        }
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        const int quarter = warp & 3;               // TMEM lanes this warp may access
        const int row_in_tile = quarter * 32 + lane;
        int nacc = 0;
        bool ok = true;
        for (int ii = 0; ii < n_my && ok; ii++) {
            Item x;
            if (!fetch_item(a, items, ii, x, threadIdx.x == 64)) continue;
            float ws[HI];
#pragma unroll
            for (int h = 0; h < HI; h++)
                ws[h] = __ldg(a.w + (int64_t)x.q * HI + h) * __ldg(a.qs + (int64_t)x.q * HI + h);
            float* srow = a.scores + (int64_t)x.q * a.ld;
            // all key scales of the item at once: one load latency per item, not per tile
            float kscales[kChunkTiles];
#pragma unroll
            for (int tt = 0; tt < kChunkTiles; tt++) {
                const int e = (x.tile0 + tt) * kTileRows + row_in_tile;
                kscales[tt] = (tt < x.ntiles && e < x.n_vis) ? __ldg(a.ks + x.row0 + e) : 0.f;
            }
#pragma unroll
            for (int tt = 0; tt < kChunkTiles; tt++) {
                if (tt >= x.ntiles) break;
                const int e = (x.tile0 + tt) * kTileRows + row_in_tile;
                const bool live = e < x.n_vis;
                const float kscale = kscales[tt];
                const int ab = nacc & 1;
                if (!mbar_wait_warp(&accfull[ab], (nacc >> 1) & 1, abort_flag, a.st)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t d[HI];
                const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(ab * HI);
                if constexpr (HI == 64) {
                    tmem_ld64(taddr, d);
                } else if constexpr (HI == 32) {
                    tmem_ld32(taddr, d);
                } else {
                    tmem_ld16(taddr, d);
                }
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&accempty[ab]);
                nacc++;
                if (live) {
                    float acc = 0.f;
#pragma unroll
                    for (int h = 0; h < HI; h++) acc = fmaf(ws[h], fmaxf(__uint_as_float(d[h]), 0.f), acc);
                    const float s = acc * kscale;
                    if (s != s) flag(a.st, CSA_DEV_NAN);
                    srow[e] = s;
                }
            }
        }
    }

    pdl_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 2 * HI < 32 ? 32 : 2 * HI);
    }
}

template <int HI>
size_t smem_bytes() {
    return 1024 + kStages * kTileBytes + 2 * HI * kDI + (2 * kStages + 9) * 8 + 16 +
           kMaxItems * sizeof(Item);
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn get_encode_fn() {
    static EncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(p);
    });
    return fn;
}

// Row-major [rows x 128] byte matrix, boxes of box_rows x 128 bytes, 128-byte swizzle.
bool make_rows_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
    EncodeFn enc = get_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)kDI, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kDI};
    const cuuint32_t box[2] = {(cuuint32_t)kDI, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

int num_sms() {
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
cudaError_t launch_hi(const uint8_t* qI, const uint8_t* kI, const IdxArgs& args,
                      cudaStream_t stream) {
    CUtensorMap mk, mq;
    if (!make_rows_map(&mk, kI, (uint64_t)args.ent_rows, kTileRows) ||
        !make_rows_map(&mq, qI, (uint64_t)args.Q * HI, HI))
        return cudaErrorInvalidValue;
    const size_t sm = smem_bytes<HI>();
    cudaError_t e = cudaFuncSetAttribute(indexer_tc_kernel<HI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    const int grid = min(args.total_items, 2 * num_sms());
    LaunchScope scope(kKIndexerTc, stream);
    return launch_pdl(indexer_tc_kernel<HI>, dim3(grid), dim3(kThreads), sm, stream, mk, mq, args);
}

}  // namespace

bool indexer_tc_supported(int HI, int dI) {
    return dI == kDI && (HI == 16 || HI == 32 || HI == 64);
}

cudaError_t launch_indexer_tc(const uint8_t* qI, const float* qs, const float* w,
                              const uint8_t* kI, const float* ks, int64_t ent_rows,
                              const int64_t* seq_len, const int64_t* ent_off,
                              const int32_t* q_seq, const int32_t* q_pos, int Q, int B, int HI,
                              int m, int max_n, float* scores, int64_t ld, int32_t* st,
                              cudaStream_t stream) {
    if (Q == 0 || max_n == 0 || ent_rows == 0) return cudaSuccess;
    IdxArgs args;
    args.qs = qs;
    args.w = w;
    args.ks = ks;
    args.seq_len = seq_len;
    args.ent_off = ent_off;
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
    args.chunks_per_q = (max_n + kChunkTiles * kTileRows - 1) / (kChunkTiles * kTileRows);
    args.total_items = Q * args.chunks_per_q;
    switch (HI) {
        case 64: return launch_hi<64>(qI, kI, args, stream);
        case 32: return launch_hi<32>(qI, kI, args, stream);
        case 16: return launch_hi<16>(qI, kI, args, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace csa
