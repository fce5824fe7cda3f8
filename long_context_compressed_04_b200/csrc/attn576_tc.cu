// Step a5 on the 5th-generation tensor cores for 576-dim compressed entries stored as
// 512 FP8 E4M3 channels (one fp32 scale per 128) + 64 BF16 RoPE channels (656-byte rows),
// with 64 or more query heads: shared-KV MQA over the selected entries plus the sliding
// window, with the attention sink and partial / inverse RoPE ("DeepSeek-V4 深度分析报告"
// 2.1 CSA and "其他注意力技术细节").
//
// One cluster of 4 CTAs per (query, group of 64 heads).  The keys of the query are tiles
// of 32 -- the window's raw rows first (RMSNormed and RoPEd here), then the selected entries
// -- dealt to the ranks in turn (tile j to rank j mod 4).  Each rank ends with an fp32
// partial state per head (running maximum, sum, unnormalised O) and stores it straight
// into the shared memory of the rank that finishes that head (16 heads each, posted
// st.shared::cluster); each rank combines its heads in rank order, the sink first.  Three
// key buffers let tiles be built while earlier ones are in the tensor cores.
//   warps 0-3  loaders: the query's 64 head rows RoPEd at t into shared memory once; per
//              tile, 4 threads per key row dequantize the gathered FP8 row (or normalise the
//              raw window row in place) into bf16, 128-byte swizzled, 9 blocks of 64
//              channels; each thread's quarter of the next entry row is loaded into
//              registers while the current tile is converted.
//   warp 4     TMEM allocation; lane 0 issues tcgen05.mma kind::f16:
//              S = Q K^T (M = 64 heads, N = 32 keys, 36 K steps of 16 channels) into one of
//              two S buffers, one tile ahead of O += P V, which goes straight into the TMEM
//              accumulator: channels 0-255 in TMEM lanes 0-15 of each quarter, 256-511 in
//              lanes 16-31, 512-575 in lanes 0-15 again (N = 256 + 256 + 64), V being the
//              key tile read MN-major.
//   warps 5-8  online softmax in the log2 domain, one head row per lane, weights by
//              ex2.approx of one FMA per key: P as bf16 into shared memory; the running
//              maximum is a reference that moves only when a tile's maximum exceeds it by
//              2^8, and then the head's O row in TMEM is rescaled; finally the partial
//              states across the cluster, and for this rank's heads the combine, the sink,
//              inverse RoPE and the store.
// A 64 x 576 fp32 accumulator takes 320 TMEM columns, and the query's Q tile (72 KB) takes a
// third of shared memory: hence 64 heads per CTA and three key buffers of 32 rows.
// All waits are bounded (timeout -> CSA_DEV_TIMEOUT, drain, free TMEM, return).  A query's
// arithmetic never depends on the batch.
#include <mutex>

#include "launchers.cuh"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kHC = 64;                  // heads per CTA (MMA M)
constexpr int kD = 576;
constexpr int kNB = kD / 64;             // 9 blocks of 64 channels (128 bytes of bf16)
constexpr int kTK = 32;                  // keys per tile (MMA N of S)
constexpr int kQBlk = 64 * 128;          // one 64-row x 128-byte swizzled block of Q
constexpr int kKBlk = kTK * 128;         // one 32-row x 128-byte swizzled block of K
constexpr int kQBytes = kNB * kQBlk;     // 72 KB
constexpr int kKBytes = kNB * kKBlk;     // 36 KB per key buffer
constexpr int kPBytes = 64 * 128;        // 8 KB (rows of 128 B, the first 64 B used)
constexpr int kRowBytes = 656;
constexpr int kThreads = 288;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.f;          // the reference maximum moves by more than 2^8 only
constexpr uint32_t kColO = 0;            // O channels 0-255 (lanes 0-15) / 256-511 (lanes 16-31)
constexpr uint32_t kColOr = 256;         // O channels 512-575 (lanes 0-15)
constexpr uint32_t kColS = 320;          // S buffers at 320 and 352 (lanes 0-15)
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxK = 2048;
constexpr int kCl = 4;                   // CTAs per (query, head group)
constexpr int kHO = kHC / kCl;           // heads finished by each rank
// shared-memory layout (byte offsets from the 1024-aligned base)
constexpr int kOffQ = 0;
constexpr int kKBuf = 3;                 // key buffers
constexpr int kOffK = kOffQ + kNB * 64 * 128;            // after Q (72 KB)
constexpr int kOffP = kOffK + kKBuf * kNB * 32 * 128;    // after the key buffers
constexpr int kOffMask = kOffP + 2 * 64 * 128;           // after two P buffers
constexpr int kOffRope = kOffMask + 16;
constexpr int kOffIdx = kOffRope + 5 * 32 * 4;
constexpr int kOffRot = kOffIdx + kMaxK * 4;              // [32 rows][32 pairs] cos, sin
constexpr int kOffWt = kOffRot + 32 * 32 * 8;              // [16 heads][kCl + 1] weights, L
constexpr int kOffBars = kOffWt + 16 * 8 * 4;
constexpr int kOffEnd = kOffBars + 22 * 8 + 16;
// the partial states of this rank's heads from every rank, [kCl][kHO][576] O then
// [kCl][2][kHO] m, l, over Q, the key, P and staging buffers once this rank's MMAs are done
constexpr int kRecvO = kCl * kHO * 576;
static_assert((kRecvO + kCl * 2 * kHO) * 4 <= kOffMask, "receive buffer");
static_assert(kOffK % 1024 == 0 && kOffP % 1024 == 0, "swizzled tiles on 1024 B");
static_assert(kOffIdx % 16 == 0 && kOffBars % 8 == 0, "alignment");

struct A576Args {
    const uint16_t* q;
    const uint8_t* entries;
    const int64_t* ent_off;
    const uint16_t* kv;
    const int64_t* kv_off;
    const int64_t* kv_pos0;
    const int32_t* q_seq;
    const int32_t* q_pos;
    const int64_t* seq_len;
    const int32_t* idx;
    const float* sink;
    uint16_t* out;
    int32_t* st;
    int64_t ent_rows;
    int k, m, B, W, H;
    float scale_log2, eps;
    double log2_theta;
};

// Byte offset of 16-byte chunk `ch` of row `r` in a 128-byte-swizzled [rows x 128 B] block.
__device__ __forceinline__ uint32_t swz(int r, int ch) {
    return (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// MN-major 128-byte-swizzled operand descriptor (rows of 128 B along MN, 8-row groups 1024 B
// apart along K; LBO = distance between 64-element MN slices).
__device__ __forceinline__ uint64_t desc_mn(const void* tile, uint32_t lbo_bytes) {
    const uint64_t addr = sm100::smem_addr(tile);
    uint64_t d = 0;
    d |= (addr >> 4) & 0x3FFFull;
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= 1ull << 46;
    d |= 2ull << 61;
    return d;
}

// 8 channels (16 bytes of bf16) of row `r`, channel `d0` (a multiple of 8), into a
// [9 blocks][rows x 128 B] swizzled tile with blocks `blk` bytes apart.
__device__ __forceinline__ uint4* cell8(uint8_t* tile, int blk, int r, int d0) {
    return reinterpret_cast<uint4*>(tile + (d0 >> 6) * blk + swz(r, (d0 & 63) >> 3));
}

// Two e4m3 codes (low 16 bits; the lower byte first) to two floats, exactly, by the packed
// hardware conversion to f16.
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint32_t two) {
    uint32_t h;
    asm("{\n\t.reg .b16 lo;\n\tcvt.u16.u32 lo, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, lo;\n\t}"
        : "=r"(h)
        : "r"(two));
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// 16 e4m3 codes times `sc`, as 16 bf16 (two 16-byte chunks).
__device__ __forceinline__ void dequant16(uint4 c, float sc, uint4& lo, uint4& hi) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    uint32_t o[8];
#pragma unroll
    for (int z = 0; z < 4; z++) {
        const float2 a = e4m3x2_to_f32x2(w[z] & 0xFFFFu);
        const float2 b = e4m3x2_to_f32x2(w[z] >> 16);
        o[2 * z] = pack_bf16x2(a.x * sc, a.y * sc);
        o[2 * z + 1] = pack_bf16x2(b.x * sc, b.y * sc);
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// One loader thread's quarter of a selected entry row: fp8 channels [128 qt, 128 qt + 128)
// with their scale, RoPE channels [16 qt, 16 qt + 16).
struct EntryQuarter {
    uint4 f[8];
    uint4 rope[2];
    float sc;
    bool valid;
};

// Loads entry v of the query's index row (staged in shared memory) into registers (flags an
// out-of-range index once per row).
__device__ __forceinline__ void fetch_entry(const A576Args& a, const int32_t* sidx, int v,
                                            int n_vis, int64_t row0, int qt, EntryQuarter& x) {
    const int e = v < a.k ? sidx[v] : -1;
    x.valid = false;
    if (e >= 0) {
        if (e < n_vis && row0 + e < a.ent_rows) {
            x.valid = true;
        } else if (qt == 0) {
            flag(a.st, CSA_DEV_OOB);
        }
    }
    if (x.valid) {
        const uint8_t* er = a.entries + (row0 + e) * (int64_t)kRowBytes;
#pragma unroll
        for (int u = 0; u < 8; u++) x.f[u] = *reinterpret_cast<const uint4*>(er + 128 * qt + 16 * u);
#pragma unroll
        for (int u = 0; u < 2; u++)
            x.rope[u] = *reinterpret_cast<const uint4*>(er + 528 + 32 * qt + 16 * u);
        x.sc = *reinterpret_cast<const float*>(er + 512 + 4 * qt);
    }
}

__global__ void __launch_bounds__(kThreads, 1) attn576_tc_kernel(const A576Args a) {
    using namespace sm100;
    constexpr uint32_t kIdescS = instr_desc(1, 1, 64, kTK);
    constexpr uint32_t kIdescPV = instr_desc(1, 1, 64, 256, 1);
    constexpr uint32_t kIdescPVr = instr_desc(1, 1, 64, 64, 1);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* sQ = smem + kOffQ;                           // [9][64 x 128 B]
    uint8_t* sK = smem + kOffK;                           // [3][9][32 x 128 B]
    uint8_t* sP = smem + kOffP;                           // [2][64 x 128 B]
    uint8_t* smask = smem + kOffMask;                     // [3][4] valid keys, 8 per warp
    float* rqc = reinterpret_cast<float*>(smem + kOffRope);   // [32] cos / sin of pair j at t
    float* rqs = rqc + 32;
    float* rf = rqs + 32;                                 // [32] frequency of pair j
    float* rwc = rf + 32;                                 // [32] cos / sin of pair j at w0
    float* rws = rwc + 32;
    int32_t* sidx = reinterpret_cast<int32_t*>(smem + kOffIdx);   // [kMaxK] the index row
    float2* srot = reinterpret_cast<float2*>(smem + kOffRot);    // window RoPE rotations
    float* swt = reinterpret_cast<float*>(smem + kOffWt);        // combine weights
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBars);
    uint64_t* qfull = bars;          // 4 loader warps
    uint64_t* kfull = bars + 1;      // [3] 4 loader warps
    uint64_t* kfree = bars + 4;      // [3] MMA commit after the tile's P V
    uint64_t* sfull = bars + 7;      // [2] MMA commit
    uint64_t* sfree = bars + 9;      // [2] 4 softmax warps
    uint64_t* pfull = bars + 11;     // [2] 4 softmax warps
    uint64_t* pfree = bars + 13;     // [2] MMA commit
    uint64_t* pvdone = bars + 15;    // MMA commit after every P V (a rescale waits for the
                                     // previous tile's: never more than one phase behind)
    uint64_t* odone = bars + 16;     // MMA commit after the last P V (one phase)
    uint64_t* drain = bars + 17;
    uint64_t* recv_ready = bars + 18;   // every rank's MMAs are done: 4 x cluster
    uint64_t* cpart_full = bars + 19;   // every rank's partials are in: 4 x cluster
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(bars + 20);
    float* recv = reinterpret_cast<float*>(smem + kOffQ);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_smem + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.H / kHC;
    const int rank = (int)cluster_ctarank();
    const int item = blockIdx.x / kCl;
    const int qi = item / G, g = item - qi * G;
    // the query (the same decision in every thread)
    const int b = a.q_seq[qi];
    const int t = a.q_pos[qi];
    const bool valid = b >= 0 && b < a.B && t >= 0 && (int64_t)t < a.seq_len[b];
    if (threadIdx.x == 0) {
        mbar_init(qfull, 4);
        for (int i = 0; i < kKBuf; i++) {
            mbar_init(&kfull[i], 4);
            mbar_init(&kfree[i], 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(&sfull[i], 1);
            mbar_init(&sfree[i], 4);
            mbar_init(&pfull[i], 4);
            mbar_init(&pfree[i], 1);
        }
        mbar_init(pvdone, 1);
        mbar_init(odone, 1);
        mbar_init(drain, 1);
        mbar_init(recv_ready, 4 * kCl);
        mbar_init(cpart_full, 4 * kCl);
        *abort_flag = 0;
        mbar_fence_init();
        if (!valid && g == 0 && rank == 0) flag(a.st, CSA_DEV_OOB);
    }
    if (threadIdx.x < 32 && valid) {
        // per query: cos / sin of every RoPE pair at t and at the window's first position
        // (angles formed and reduced in fp64), and the pair frequencies
        const int w0q = t - a.W + 1 > 0 ? t - a.W + 1 : 0;
        float cs, sn;
        rope_cos_sin((double)t, threadIdx.x, a.log2_theta, cs, sn);
        rqc[threadIdx.x] = cs;
        rqs[threadIdx.x] = sn;
        rope_cos_sin((double)w0q, threadIdx.x, a.log2_theta, cs, sn);
        rwc[threadIdx.x] = cs;
        rws[threadIdx.x] = sn;
        rf[threadIdx.x] = (float)exp2(-(double)(2 * threadIdx.x) * (1.0 / 64.0) * a.log2_theta);
    }
    if (warp == 4) {
        tmem_alloc(tmem_base_smem, kTmemCols);
        tmem_relinquish();
    }
    // the index sets come from the top-k and the entries from compression
    pdl_wait();
    if (threadIdx.x == 0) pdl_trigger();
    if (valid) {
        // the query's index row, once (only the loaders read it)
        for (int v = threadIdx.x; v < a.k; v += kThreads) sidx[v] = a.idx[(int64_t)qi * a.k + v];
    }
    tc_fence_before();
    __syncthreads();
    // the cluster's barriers are initialised before any rank arrives on another's
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;

    const int n_vis = valid ? (t + 1) / a.m : 0;
    const int64_t row0 = valid ? a.ent_off[b] : 0;
    const int w0 = t - a.W + 1 > 0 ? t - a.W + 1 : 0;
    const int n_win = a.W > 0 ? t - w0 + 1 : 0;
    const int n_wt = (a.W + kTK - 1) / kTK;          // window tiles (masked past n_win)
    const int n_et = (a.k + kTK - 1) / kTK;          // selected-entry tiles
    const int ntiles = valid ? n_wt + n_et : 0;
    // this rank's tiles: global tile rank + kCl j for local j < nloc
    const int nloc = ntiles > rank ? (ntiles - rank + kCl - 1) / kCl : 0;

    if (warp < 4) {
        // ---------------- loaders ----------------
        const int tid = threadIdx.x;
        const int r = tid >> 1, hf = tid & 1;        // key (or head) row, half of it
        bool ok = true;
        if (valid) {
            // q head row r at t: channels [288 hf, 288 hf + 288), RoPE on 512..575
            const uint16_t* qrow = a.q + ((int64_t)qi * a.H + kHC * g + r) * kD;
#pragma unroll
            for (int half = 0; half < 2; half++) {
                uint4 u[18];   // 18 loads in flight
#pragma unroll
                for (int c = 0; c < 18; c++)
                    u[c] = *reinterpret_cast<const uint4*>(qrow + 288 * hf + 144 * half + 8 * c);
#pragma unroll
                for (int c = 0; c < 18; c++) {
                    const int d0 = 288 * hf + 144 * half + 8 * c;
                    if (d0 >= kD - kRopeDims) {
                        uint32_t w[4] = {u[c].x, u[c].y, u[c].z, u[c].w};
#pragma unroll
                        for (int z = 0; z < 4; z++) {
                            const int pj = (d0 - (kD - kRopeDims)) / 2 + z;
                            const float2 f = bf16x2_to_f32(w[z]);
                            w[z] = pack_bf16x2(f.x * rqc[pj] - f.y * rqs[pj], f.x * rqs[pj] + f.y * rqc[pj]);
                        }
                        u[c] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                    *cell8(sQ, kQBlk, r, d0) = u[c];
                }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(qfull);
        }
        // tiles: 4 threads per key row, quarter qt
        const int kr = tid >> 2, qt = tid & 3;
        EntryQuarter ex;
        ex.valid = false;
        if (nloc > 0 && rank >= n_wt) fetch_entry(a, sidx, (rank - n_wt) * kTK + kr, n_vis, row0, qt, ex);
        for (int j = 0; j < nloc && ok; j++) {
            const int jg = rank + kCl * j;   // global tile
            const int kb = j % kKBuf;
            uint8_t* tile = sK + kb * kKBytes;
            // this key buffer is free once the P V of the tile kKBuf back has completed
            if (!mbar_wait_warp(&kfree[kb], ((j / kKBuf) & 1) ^ 1, abort_flag, a.st)) {
                ok = false;
                break;
            }
            bool vrow;
            if (jg < n_wt) {
                // window row: RMSNorm over all 576 channels (the four quarters meet by
                // shuffle), RoPE at its own position on 512..575
                const int wr = jg * kTK + kr;
                const int64_t p = (int64_t)w0 + wr;
                vrow = wr < n_win;
                if (vrow && p < a.kv_pos0[b]) {
                    vrow = false;
                    if (qt == 0) flag(a.st, CSA_DEV_OOB);
                }
                const uint16_t* src =
                    vrow ? a.kv + (a.kv_off[b] + p - a.kv_pos0[b]) * (int64_t)kD : nullptr;
                // pass 1: my quarter of the raw row into the tile (18 loads in flight) and its
                // sum of squares
                float ss = 0.f;
                {
                    uint4 u[18];
#pragma unroll
                    for (int c = 0; c < 18; c++)
                        u[c] = vrow ? *reinterpret_cast<const uint4*>(src + 144 * qt + 8 * c)
                                    : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int c = 0; c < 18; c++) {
                        const uint32_t w[4] = {u[c].x, u[c].y, u[c].z, u[c].w};
#pragma unroll
                        for (int z = 0; z < 4; z++) {
                            const float2 f = bf16x2_to_f32(w[z]);
                            ss += f.x * f.x + f.y * f.y;
                        }
                        *cell8(tile, kKBlk, kr, 144 * qt + 8 * c) = u[c];
                    }
                }
                ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                ss += __shfl_xor_sync(0xffffffffu, ss, 2);
                const float rn = rsqrtf(ss / (float)kD + a.eps);
                // rotations of the tile's 32 rows x 32 pairs, 8 per loader thread:
                // angle (w0 + wr) f_j = w0 f_j (fp64 table) + wr f_j (< 128 rad, sincosf),
                // combined by the addition formula
#pragma unroll 1
                for (int e = tid; e < kTK * 32; e += 128) {
                    const int er = e >> 5, pj = e & 31;
                    float sb_, cb_;
                    sincosf((float)(jg * kTK + er) * rf[pj], &sb_, &cb_);
                    srot[e] = make_float2(rwc[pj] * cb_ - rws[pj] * sb_, rws[pj] * cb_ + rwc[pj] * sb_);
                }
                asm volatile("bar.sync 3, 128;" ::: "memory");
                // pass 2, in place in shared memory: normalise, RoPE at the row's position
                if (vrow) {
#pragma unroll 3
                    for (int c = 0; c < 18; c++) {
                        const int d0 = 144 * qt + 8 * c;
                        uint4* cl = cell8(tile, kKBlk, kr, d0);
                        const uint4 u = *cl;
                        const uint32_t wi[4] = {u.x, u.y, u.z, u.w};
                        uint32_t w[4];
#pragma unroll
                        for (int z = 0; z < 4; z++) {
                            float2 f = bf16x2_to_f32(wi[z]);
                            f.x *= rn;
                            f.y *= rn;
                            if (d0 >= kD - kRopeDims) {
                                const float2 cs = srot[kr * 32 + (d0 - (kD - kRopeDims)) / 2 + z];
                                f = make_float2(f.x * cs.x - f.y * cs.y, f.x * cs.y + f.y * cs.x);
                            }
                            w[z] = pack_bf16x2(f.x, f.y);
                        }
                        *cl = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
                // every loader is done with this tile's rotations before the next tile's
                asm volatile("bar.sync 3, 128;" ::: "memory");
            } else {
                vrow = ex.valid;
#pragma unroll
                for (int u = 0; u < 8; u++) {
                    uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
                    if (vrow) dequant16(ex.f[u], ex.sc, lo, hi);
                    const int d0 = 128 * qt + 16 * u;
                    *cell8(tile, kKBlk, kr, d0) = lo;
                    *cell8(tile, kKBlk, kr, d0 + 8) = hi;
                }
#pragma unroll
                for (int u = 0; u < 2; u++)
                    *cell8(tile, kKBlk, kr, 512 + 16 * qt + 8 * u) = vrow ? ex.rope[u] : make_uint4(0u, 0u, 0u, 0u);
            }
            // valid keys of the tile: this warp's 8 rows (lanes 0, 4, ..., 28 carry them)
            const uint32_t bal = __ballot_sync(0xffffffffu, vrow && qt == 0);
            uint32_t m8 = 0;
#pragma unroll
            for (int i = 0; i < 8; i++) m8 |= ((bal >> (4 * i)) & 1u) << i;
            if (lane == 0) smask[kb * 4 + warp] = (uint8_t)m8;
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&kfull[kb]);
            // the next entry tile's rows in flight while this one is used
            if (j + 1 < nloc && jg + kCl >= n_wt)
                fetch_entry(a, sidx, (jg + kCl - n_wt) * kTK + kr, n_vis, row0, qt, ex);
        }
    } else if (warp == 4) {
        if (lane == 0 && nloc > 0) {
            // ---------------- MMA issuer ----------------
            // S of a tile is issued before the P V of the previous one, so the softmax of
            // one tile overlaps the tensor work of its neighbours
            bool ok = mbar_wait(qfull, 0, abort_flag, a.st);
            tc_fence_after();
            auto issue_s = [&](int j) -> bool {
                const int kb = j % kKBuf, sb = j & 1;
                if (!mbar_wait(&kfull[kb], (j / kKBuf) & 1, abort_flag, a.st) ||
                    !mbar_wait(&sfree[sb], ((j >> 1) & 1) ^ 1, abort_flag, a.st))
                    return false;
                tc_fence_after();
                const uint32_t ds = tmem + kColS + (uint32_t)(sb * kTK);
                const uint8_t* tile = sK + kb * kKBytes;
#pragma unroll 1
                for (int cb = 0; cb < kNB; cb++) {
                    const uint64_t ad = smem_desc_k_sw128(sQ + cb * kQBlk);
                    const uint64_t bd = smem_desc_k_sw128(tile + cb * kKBlk);
#pragma unroll
                    for (int kk = 0; kk < 4; kk++)   // K = 16 bf16 = 32 bytes per MMA
                        mma_f16(ds, ad + 2 * kk, bd + 2 * kk, kIdescS, (cb | kk) ? 1u : 0u);
                }
                mma_commit(&sfull[sb]);
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int j = 0; j < nloc && ok; j++) {
                if (j + 1 < nloc && !issue_s(j + 1)) {
                    ok = false;
                    break;
                }
                const int kb = j % kKBuf, sb = j & 1;
                if (!mbar_wait(&pfull[sb], (j >> 1) & 1, abort_flag, a.st)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t pa = smem_desc_k_sw128(sP + sb * kPBytes);
                const uint8_t* tile = sK + kb * kKBytes;
#pragma unroll
                for (int kk = 0; kk < kTK / 16; kk++) {   // 16 keys per MMA
                    const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
                    mma_f16(tmem + kColO, pa + 2 * kk, desc_mn(tile + kk * 2048, kKBlk), kIdescPV, acc);
                    mma_f16(tmem + kColO + (16u << 16), pa + 2 * kk,
                            desc_mn(tile + 4 * kKBlk + kk * 2048, kKBlk), kIdescPV, acc);
                    mma_f16(tmem + kColOr, pa + 2 * kk, desc_mn(tile + 8 * kKBlk + kk * 2048, kKBlk),
                            kIdescPVr, acc);
                }
                mma_commit(&kfree[kb]);
                mma_commit(&pfree[sb]);
                mma_commit(pvdone);
            }
            if (ok) mma_commit(odone);
            // drain: all issued MMAs complete before TMEM is released
            mma_commit(drain);
            mbar_drain(drain, 0, a.st);
        }
    } else {
        // ---------------- softmax / epilogue (warps 5..8) ----------------
        const int quarter = warp & 3;
        const int hl = quarter * 16 + (lane & 15);   // head within the group
        const bool mine = lane < 16;                 // S rows live in lanes 0-15
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        float mref = -INFINITY, lrun = 0.f;
        bool ok = true;
        for (int j = 0; j < nloc && ok; j++) {
            const int sb = j & 1;
            if (!mbar_wait_warp(&sfull[sb], (j >> 1) & 1, abort_flag, a.st)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sv[kTK];
            tmem_ld32(tmem + kColS + (uint32_t)(sb * kTK) + lane_base, sv);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sfree[sb]);
            const uint8_t* mk = smask + (j % kKBuf) * 4;
            const uint32_t mbits = (uint32_t)mk[0] | ((uint32_t)mk[1] << 8) |
                                   ((uint32_t)mk[2] << 16) | ((uint32_t)mk[3] << 24);
            // raw scores (masked keys -inf); the scale is positive, so the maximum of the
            // scaled scores is the scaled maximum
            const uint32_t mon = mine ? mbits : 0u;
            float rmax = -INFINITY;
            if (mon == 0xffffffffu) {
#pragma unroll
                for (int c = 0; c < kTK; c++) rmax = fmaxf(rmax, __uint_as_float(sv[c]));
            } else {
#pragma unroll
                for (int c = 0; c < kTK; c++) {
                    const float xv = ((mon >> c) & 1u) ? __uint_as_float(sv[c]) : -INFINITY;
                    sv[c] = __float_as_uint(xv);
                    rmax = fmaxf(rmax, xv);
                }
            }
            const float tmax = rmax * a.scale_log2;
            // move the reference maximum only on a jump of more than 2^8
            const bool need = mine && tmax > mref + kRescale;
            if (__any_sync(0xffffffffu, need)) {
                const float mnew = need ? tmax : mref;
                const float corr = (!need || mref == -INFINITY) ? (need ? 0.f : 1.f)
                                                                 : exp2f(mref - mnew);
                if (j > 0) {
                    // the running O must be complete before its rows are rescaled
                    if (!mbar_wait_warp(pvdone, (j - 1) & 1, abort_flag, a.st)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const float f = __shfl_sync(0xffffffffu, corr, lane & 15);
                    if (__any_sync(0xffffffffu, f != 1.f)) {
#pragma unroll 1
                        for (int cc = 0; cc < 20; cc++) {
                            // 16 columns at a time: 0-255 (both lane halves), then 256-319
                            const uint32_t col = cc < 16 ? kColO + 16u * cc : kColOr + 16u * (cc - 16);
                            uint32_t ov[16];
                            tmem_ld16(tmem + col + lane_base, ov);
                            tmem_ld_wait();
#pragma unroll
                            for (int z = 0; z < 16; z++) ov[z] = __float_as_uint(__uint_as_float(ov[z]) * f);
                            tmem_st16(tmem + col + lane_base, ov);
                        }
                        tmem_st_wait();
                    }
                    tc_fence_before();
                }
                lrun *= corr;
                mref = mnew;
            }
            // P = 2^(s * scale - mref): one FMA and one ex2 per key (a masked key is -inf,
            // giving 0); with no valid key yet (mref = -inf) every P of the tile is 0
            float rs = 0.f;
            uint32_t pk[kTK / 2];
            if (mref == -INFINITY) {
#pragma unroll
                for (int c = 0; c < kTK / 2; c++) pk[c] = 0u;
            } else {
                const float nm = -mref;
#pragma unroll
                for (int c = 0; c < kTK / 2; c++) {
                    const float p0 = ex2_approx(fmaf(__uint_as_float(sv[2 * c]), a.scale_log2, nm));
                    const float p1 = ex2_approx(fmaf(__uint_as_float(sv[2 * c + 1]), a.scale_log2, nm));
                    rs += p0 + p1;
                    pk[c] = pack_bf16x2(p0, p1);
                }
            }
            lrun += rs;
            if (!mbar_wait_warp(&pfree[sb], ((j >> 1) & 1) ^ 1, abort_flag, a.st)) {
                ok = false;
                break;
            }
            if (mine) {
                uint8_t* prow = sP + sb * kPBytes;
#pragma unroll
                for (int c = 0; c < kTK / 8; c++)
                    *reinterpret_cast<uint4*>(prow + swz(hl, c)) =
                        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pfull[sb]);
        }
        if (ok && nloc > 0) ok = mbar_wait_warp(odone, 0, abort_flag, a.st);
        if (ntiles > 0) {
            // ---- partial states across the cluster ----
            // my MMAs are done: my Q / key / P / staging buffers may take the partials
            if (ok) {
                tc_fence_after();
                __syncwarp();
                if (lane == 0)
                    for (int rr = 0; rr < kCl; rr++) mbar_arrive_cluster(mapa(recv_ready, (uint32_t)rr));
                ok = mbar_wait_cluster_warp(recv_ready, 0, abort_flag, a.st);
            }
            if (ok) {
                // head hl goes to rank hl / kHO (this warp's 16 heads: rank `quarter`)
                const int own = hl / kHO, lh = hl - own * kHO;
                float* recv_ml = recv + kRecvO;
                const uint32_t dst = mapa(recv + (rank * kHO + lh) * 576 + (mine ? 0 : 256), (uint32_t)own);
#pragma unroll 1
                for (int cc = 0; cc < 5; cc++) {
                    // 64 columns at a time: 0-255 (both lane halves), then 256-319 (lanes 0-15)
                    const uint32_t col = cc < 4 ? kColO + 64u * cc : kColOr;
                    uint32_t ov[64];
                    if (nloc > 0) {
                        tmem_ld64(tmem + col + lane_base, ov);
                        tmem_ld_wait();
                    } else {
#pragma unroll
                        for (int z = 0; z < 64; z++) ov[z] = 0u;
                    }
                    if (cc < 4 || mine) {
                        // lanes 0-15: channels 0-255 then 512-575; lanes 16-31: 256-511
                        const uint32_t off = (cc < 4 ? 64u * cc : 512u) * 4u;
#pragma unroll
                        for (int z = 0; z < 64; z += 4)
                            st_cluster_f4(dst + off + 4u * z,
                                          make_float4(__uint_as_float(ov[z]), __uint_as_float(ov[z + 1]),
                                                      __uint_as_float(ov[z + 2]), __uint_as_float(ov[z + 3])));
                    }
                }
                if (mine) {
                    st_cluster_f32(mapa(recv_ml + (2 * rank) * kHO + lh, (uint32_t)own), mref);
                    st_cluster_f32(mapa(recv_ml + (2 * rank + 1) * kHO + lh, (uint32_t)own), lrun);
                }
                tc_fence_before();
                fence_cluster();
                __syncwarp();
                if (lane == 0)
                    for (int rr = 0; rr < kCl; rr++) mbar_arrive_cluster(mapa(cpart_full, (uint32_t)rr));
                ok = mbar_wait_cluster_warp(cpart_full, 0, abort_flag, a.st);
            }
            if (named_barrier_and(2, 128, ok)) {
                // this rank's heads; first the combine weights, one thread per head:
                // M = max(sink, m_r), w_r = 2^(m_r - M), L = 2^(sink - M) + sum_r w_r l_r
                const float* recv_ml = recv + kRecvO;
                const int i = threadIdx.x - 160;
                if (i < kHO) {
                    const float sk = a.sink[kHC * g + rank * kHO + i] * kLog2e;
                    float M = sk;
#pragma unroll
                    for (int rr = 0; rr < kCl; rr++) M = fmaxf(M, recv_ml[(2 * rr) * kHO + i]);
                    float L = (M == -INFINITY || sk == -INFINITY) ? 0.f : exp2f(sk - M);
#pragma unroll
                    for (int rr = 0; rr < kCl; rr++) {
                        const float mr = recv_ml[(2 * rr) * kHO + i];
                        const float wgt = (mr == -INFINITY) ? 0.f : exp2f(mr - M);
                        L = fmaf(wgt, recv_ml[(2 * rr + 1) * kHO + i], L);
                        swt[i * 8 + rr] = wgt;
                    }
                    swt[i * 8 + kCl] = L;
                }
                asm volatile("bar.sync 2, 128;" ::: "memory");
                // then (head, 4 channels) per work unit: sum_r w_r O_r / L
#pragma unroll 2
                for (int w = i; w < kHO * (576 / 4); w += 128) {
                    const int lh = w / (576 / 4), c4 = (w - lh * (576 / 4)) * 4;
                    const int h = kHC * g + rank * kHO + lh;
                    const float L = swt[lh * 8 + kCl];
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int rr = 0; rr < kCl; rr++) {
                        const float wgt = swt[lh * 8 + rr];
                        const float4 v = *reinterpret_cast<const float4*>(recv + (rr * kHO + lh) * 576 + c4);
                        acc.x = fmaf(wgt, v.x, acc.x);
                        acc.y = fmaf(wgt, v.y, acc.y);
                        acc.z = fmaf(wgt, v.z, acc.z);
                        acc.w = fmaf(wgt, v.w, acc.w);
                    }
                    if (L > 0.f) {
                        acc.x /= L;
                        acc.y /= L;
                        acc.z /= L;
                        acc.w /= L;
                    } else {
                        acc = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                    if (c4 >= kD - kRopeDims) {
                        // rotation by -t: (x, y) -> (x cos + y sin, y cos - x sin)
                        const int pj = (c4 - (kD - kRopeDims)) >> 1;
                        const float c0 = rqc[pj], s0 = rqs[pj], c1 = rqc[pj + 1], s1 = rqs[pj + 1];
                        acc = make_float4(acc.x * c0 + acc.y * s0, acc.y * c0 - acc.x * s0,
                                          acc.z * c1 + acc.w * s1, acc.w * c1 - acc.z * s1);
                    }
                    *reinterpret_cast<uint2*>(a.out + ((int64_t)qi * a.H + h) * kD + c4) =
                        make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    // no rank leaves while another may still store into its shared memory
    cluster_sync_all();
}

static_assert(kOffK == kQBytes && kOffP == kOffK + kKBuf * kKBytes &&
                  kOffMask == kOffP + 2 * kPBytes,
              "layout");
constexpr size_t kSmemBytes = 1024 + kOffEnd;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

}  // namespace

bool attn576_tc_supported(int H, int D, int fmt) {
    return D == kD && fmt == CSA_KV_FP8_576 && H % kHC == 0;
}

cudaError_t launch_attn576_tc(const AttnArgs& aa, int Q, cudaStream_t stream) {
    if (Q == 0) return cudaSuccess;
    A576Args a;
    a.q = aa.q;
    a.entries = aa.entries;
    a.ent_off = aa.ent_off;
    a.kv = aa.kv;
    a.kv_off = aa.kv_off;
    a.kv_pos0 = aa.kv_pos0;
    a.q_seq = aa.q_seq;
    a.q_pos = aa.q_pos;
    a.seq_len = aa.seq_len;
    a.idx = aa.idx;
    a.sink = aa.sink;
    a.out = aa.out;
    a.st = aa.st;
    a.ent_rows = aa.ent_rows;
    a.k = aa.k;
    a.m = aa.m;
    a.B = aa.B;
    a.W = aa.W;
    a.H = aa.H;
    a.scale_log2 = aa.scale * kLog2e;
    a.eps = aa.eps;
    a.log2_theta = aa.log2_theta;
    cudaError_t e = cudaFuncSetAttribute(attn576_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    LaunchScope scope(kKAttn576Tc, stream);
    return launch_pdl_cluster(attn576_tc_kernel, dim3(Q * (aa.H / kHC) * kCl), dim3(kThreads),
                              kSmemBytes, stream, kCl, a);
}

}  // namespace csa
