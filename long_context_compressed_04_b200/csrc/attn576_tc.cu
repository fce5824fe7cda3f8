// Step a5 on the 5th-generation tensor cores for 576-dim compressed entries stored as
// 512 FP8 E4M3 channels (one fp32 scale per 128) + 64 BF16 RoPE channels (656-byte rows),
// with 64 or more query heads: shared-KV MQA over the selected entries plus the sliding
// window, with the attention sink and partial / inverse RoPE ("DeepSeek-V4 深度分析报告"
// 2.1 CSA and "其他注意力技术细节").
//
// One cluster of 4 CTAs per (query, group of 64 heads).  The keys of the query are tiles
// of 32 -- the window's raw rows first (RMSNormed and RoPEd here), then the selected entries
// -- dealt to the ranks in turn (tile j to rank j mod 4, so every rank's first tile is a
// window tile).  The query tile and the window tile depend only on the call's inputs, so
// they are built, scored and accumulated before the kernel waits for the one before it
// (the top-k): only the index row and the entries wait.  Each rank ends with an fp32
// partial state per head (running maximum, sum, unnormalised O) in its own shared memory;
// the rank that finishes a head pulls the four partial states of it (ld.shared::cluster)
// and combines them in rank order, the sink first.  Three key buffers let tiles be built
// while earlier ones are in the tensor cores.
//   warps 0-3  loaders: the query's 64 head rows RoPEd at t into shared memory once (as
//              fp16, scaled by 2^-s if needed, see below); the window tile; then, after the
//              wait, the index row; per tile, 4 threads per key row convert their quarter
//              of the FP8 row (16 channels of every 64, so that a warp load reads 64
//              contiguous bytes of each of 8 rows; e4m3 -> fp16 exactly, times the block
//              scale) into a 128-byte-swizzled tile of 9 blocks of 64 channels; the rows of
//              tile j + 2 are loaded into registers while tile j is converted (two
//              register sets).
//   warp 4     TMEM allocation; lane 0 issues O += P V (tcgen05.mma kind::f16, fp16
//              operands) straight into the TMEM accumulator: channels 0-255 in TMEM lanes
//              0-15 of each quarter, 256-511 in lanes 16-31, 512-575 in lanes 0-15 again
//              (N = 256 + 256 + 64), V being the key tile read MN-major.
//   warps 9-10 lane 0 issues S = Q K^T of every tile (M = 64 heads, N = 32 keys, 36 K
//              steps of 16 channels) into S buffer j % 2 as 4 partial accumulators (see
//              s_col), warp 9 partials 0 and 2, warp 10 partials 1 and 3: one MMA costs its
//              issuing thread tens of cycles whatever its shape, so S has two issuers, and
//              both on one tile halve its latency.
//   warps 5-8  online softmax in the log2 domain, one head row per lane, weights by
//              ex2.approx of one FMA per key: P as fp16 into shared memory; the running
//              maximum is a reference that moves only when a tile's maximum exceeds it by
//              2^8, and then the head's O row in TMEM is rescaled; then the partial state
//              into shared memory.
//   warps 0-3, 5-8  the combine of this rank's 16 heads: inverse RoPE, bf16 store.
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
constexpr int kNB = kD / 64;             // 9 blocks of 64 channels (128 bytes of fp16)
constexpr int kTK = 32;                  // keys per tile (MMA N of S)
constexpr int kQBlk = 64 * 128;          // one 64-row x 128-byte swizzled block of Q
constexpr int kKBlk = kTK * 128;         // one 32-row x 128-byte swizzled block of K
constexpr int kQBytes = kNB * kQBlk;     // 72 KB
constexpr int kKBytes = kNB * kKBlk;     // 36 KB per key buffer
constexpr int kPBytes = 64 * 128;        // 8 KB (rows of 128 B, the first 64 B used)
constexpr int kRowBytes = 656;
constexpr int kFirstSWarp = 9;           // warps 9 and 10 issue S (see the MMA issuers)
constexpr int kThreads = 32 * (kFirstSWarp + 2);
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.f;          // the reference maximum moves by more than 2^8 only
constexpr uint32_t kColO = 0;            // O channels 0-255 (lanes 0-15) / 256-511 (lanes 16-31)
constexpr uint32_t kColOr = 256;         // O channels 512-575 (lanes 0-15)
constexpr uint32_t kColS = 320;          // S: [2 buffers][4 partials] x 32 columns, see s_col
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxK = 2048;
constexpr int kCl = 4;                   // CTAs per (query, head group)
constexpr int kHO = kHC / kCl;           // heads finished by each rank
constexpr int kWtStride = kCl + 1;       // combine weights of a head: kCl ranks, then L
static_assert(kCl >= 4, "the window (at most 4 tiles of 32 rows) is one tile per rank");
// shared-memory layout (byte offsets from the 1024-aligned base)
constexpr int kOffQ = 0;
constexpr int kKBuf = 3;                 // key buffers (fp16)
constexpr int kOffK = kOffQ + kNB * 64 * 128;            // after Q (72 KB)
constexpr int kOffP = kOffK + kKBuf * kNB * 32 * 128;    // after the key buffers
constexpr int kOffMask = kOffP + 2 * 64 * 128;           // after two P buffers
constexpr int kOffRope = kOffMask + 16;   // [kKBuf][4] key masks
constexpr int kOffQMax = kOffRope + 5 * 32 * 4;       // [4] per-warp max |q|, then the q scale
constexpr int kOffIdx = kOffQMax + 32;
constexpr int kOffRot = kOffIdx + kMaxK * 4;              // [32 rows][32 pairs] cos, sin
constexpr int kOffWt = kOffRot + 32 * 32 * 8;              // [16 heads][kCl + 1] weights, L
constexpr int kOffBars = kOffWt + 16 * 8 * 4;
static_assert(kHO * kWtStride <= 16 * 8, "combine-weight table");
constexpr int kOffEnd = kOffBars + 21 * 8 + 16;
// this rank's partial state, written over Q / K / P once its MMAs are done and read by the
// rank that finishes each head: O as [64 heads][kPS] fp32 (rows padded from 576 to 580
// floats, so that the lanes writing 16 head rows at once hit distinct banks), then the
// running maximum m [64] and sum l [64]
constexpr int kPS = 580;
constexpr int kPartML = kHC * kPS;
static_assert((kPartML + 2 * kHC) * 4 <= kOffMask, "partial state over Q / K / P");
static_assert(kOffK % 1024 == 0 && kOffP % 1024 == 0, "swizzled tiles on 1024 B");
static_assert(kOffIdx % 16 == 0 && kOffBars % 8 == 0, "alignment");

struct A576Args {
    const uint16_t* q;
    const uint8_t* entries;
    EntryRows er;
    const uint16_t* kv;
    RawRows raw;
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

// S of a key tile is accumulated in 4 independent partials, partial p taking the K steps
// 4 cb + p (cb = the 64-channel block): a chain of MMAs into one accumulator waits for each
// step's result, four chains keep the tensor pipe busy.  Partial p of S buffer sb sits at
// columns kColS + 32 (2 sb + p / 2), in TMEM lanes 0-15 (p even) or 16-31 (p odd) of each
// lane quarter (an M = 64 accumulator uses 16 lanes per quarter).
__host__ __device__ constexpr uint32_t s_col(int sb, int p) {
    return kColS + 32u * (uint32_t)(2 * sb + (p >> 1)) + ((uint32_t)(p & 1) << 20);
}
static_assert(s_col(1, 3) - (16u << 16) + 32 <= kTmemCols, "S partials fit the allocation");

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

// 8 channels (16 bytes of fp16) of row `r`, channel `d0` (a multiple of 8), into a
// [9 blocks][rows x 128 B] swizzled tile with blocks `blk` bytes apart.
__device__ __forceinline__ uint4* cell8(uint8_t* tile, int blk, int r, int d0) {
    return reinterpret_cast<uint4*>(tile + (d0 >> 6) * blk + swz(r, (d0 & 63) >> 3));
}

// The MMAs of this kernel take fp16 operands (Q, K = V and P; fp32 accumulation).  An e4m3
// code is exact in fp16, so an entry channel is one conversion and one multiply by its
// block's scale (rounded to fp16); entries and window rows are RMS-normalised (|x| <= sqrt(D)),
// and fp16 keeps 3 more mantissa bits than bf16.  The query is scaled by an exact power of
// two when its magnitude would leave the fp16 range (see the query load).

// Two floats to packed fp16 (round to nearest even; the first in the low half).
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Two e4m3 codes (low 16 bits; the lower byte first) to packed fp16, exactly.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
    uint32_t h;
    asm("{\n\t.reg .b16 lo;\n\tcvt.u16.u32 lo, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, lo;\n\t}"
        : "=r"(h)
        : "r"(two));
    return h;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t x, uint32_t y) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(y));
    return r;
}

// 16 e4m3 codes times the scale `sc2` (fp16, in both halves), as 16 fp16 (two 16-byte chunks).
__device__ __forceinline__ void dequant16(uint4 c, uint32_t sc2, uint4& lo, uint4& hi) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    uint32_t o[8];
#pragma unroll
    for (int z = 0; z < 4; z++) {
        o[2 * z] = hmul2(e4m3x2_to_f16x2(w[z] & 0xFFFFu), sc2);
        o[2 * z + 1] = hmul2(e4m3x2_to_f16x2(w[z] >> 16), sc2);
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// One loader thread's quarter of a selected entry row, in registers: the fp8 channels
// [64 u + 16 qt, 64 u + 16 qt + 16) for u = 0..7, the row's four block scales, and the RoPE
// channels [16 qt, 16 qt + 16).  The four threads of a row read 64 contiguous bytes per
// load, so one warp load touches 8 lines (of the warp's 8 rows) rather than 32.
struct EntryQuarter {
    uint4 f[8];
    uint4 rope[2];
    float4 sc;
    bool valid;
};

// Issues the loads of entry v of the query's index row (staged in shared memory) into
// registers (flags an out-of-range index once per row).
__device__ __forceinline__ void fetch_entry(const A576Args& a, const int32_t* sidx, int v,
                                            int n_vis, int b, int64_t row0, int qt,
                                            EntryQuarter& x) {
    const int e = v < a.k ? sidx[v] : -1;
    x.valid = false;
    int64_t re = 0;
    if (e >= 0) {
        re = a.er.bt ? (e < n_vis ? a.er.row(b, e) : -1) : row0 + e;
        if (e < n_vis && re >= 0 && re < a.ent_rows) {
            x.valid = true;
        } else if (qt == 0) {
            flag(a.st, CSA_DEV_OOB);
        }
    }
    if (x.valid) {
        const uint8_t* er = a.entries + re * (int64_t)kRowBytes;
#pragma unroll
        for (int u = 0; u < 8; u++) x.f[u] = *reinterpret_cast<const uint4*>(er + 64 * u + 16 * qt);
#pragma unroll
        for (int u = 0; u < 2; u++)
            x.rope[u] = *reinterpret_cast<const uint4*>(er + 528 + 32 * qt + 16 * u);
        x.sc = *reinterpret_cast<const float4*>(er + 512);
    }
}

__global__ void __launch_bounds__(kThreads, 1) attn576_tc_kernel(const A576Args a) {
    using namespace sm100;
    constexpr uint32_t kIdescS = instr_desc(0, 0, 64, kTK);         // fp16 x fp16 -> fp32
    constexpr uint32_t kIdescPV = instr_desc(0, 0, 64, 256, 1);
    constexpr uint32_t kIdescPVr = instr_desc(0, 0, 64, 64, 1);
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
    uint32_t* qmax = reinterpret_cast<uint32_t*>(smem + kOffQMax);   // [4] largest |q| bits
    float* qscale = reinterpret_cast<float*>(smem + kOffQMax + 16);   // 2^s of the q scaling
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
    uint64_t* cpart_full = bars + 19;   // every rank's partial state is written: 4 x cluster
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(bars + 20);
    float* part = reinterpret_cast<float*>(smem + kOffQ);          // [64][kPS] O, m[64], l[64]
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
            mbar_init(&sfull[i], 2);   // both S issuers commit every tile
            mbar_init(&sfree[i], 4);
            mbar_init(&pfull[i], 4);
            mbar_init(&pfree[i], 1);
        }
        mbar_init(pvdone, 1);
        mbar_init(odone, 1);
        mbar_init(drain, 3);   // the three MMA issuers

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
    // Nothing up to the loaders' wait below reads what an earlier libcsa kernel writes: the
    // query's heads, the window's raw rows and the sink are inputs.  So the query tile and
    // the window tile (S, softmax and P V included) overlap the kernel before this one (the
    // top-k); only the index row and the entries it selects wait for it.
    tc_fence_before();
    __syncthreads();
    // the cluster's barriers are initialised before any rank arrives on another's
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;

    const int n_vis = valid ? (t + 1) / a.m : 0;
    const int64_t row0 = valid && !a.er.bt ? a.er.ent_off[b] : 0;
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
        // A rank without tiles needs no Q tile; its softmax warps write its (empty) partial
        // state over Q / K at once, so nothing else may be written there.
        if (valid && nloc > 0) {
            // q head row r at t: channels [288 hf, 288 hf + 288), RoPE on 512..575.  Pass 1:
            // the largest |q| of the CTA's 64 heads; if it could leave the fp16 range after
            // the rotation (which grows a pair's component by at most sqrt 2), every q value
            // is scaled by 2^-s (exact) with s the least such that max |q| 2^-s < 2^15, and
            // the softmax scale is multiplied by 2^s.  Pass 2: rotate, scale, store as fp16.
            const uint16_t* qrow = a.q + ((int64_t)qi * a.H + kHC * g + r) * kD + 288 * hf;
            uint32_t mx = 0;   // largest |q| as bf16 bits (the order of non-negative values)
#pragma unroll
            for (int half = 0; half < 2; half++) {
                uint4 u[18];
#pragma unroll
                for (int c = 0; c < 18; c++) u[c] = *reinterpret_cast<const uint4*>(qrow + 144 * half + 8 * c);
#pragma unroll
                for (int c = 0; c < 18; c++) {
                    const uint32_t w[4] = {u[c].x, u[c].y, u[c].z, u[c].w};
#pragma unroll
                    for (int z = 0; z < 4; z++)
                        mx = max(mx, max(w[z] & 0x7FFFu, (w[z] >> 16) & 0x7FFFu));
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (lane == 0) qmax[warp] = mx;
            asm volatile("bar.sync 3, 128;" ::: "memory");
            mx = max(max(qmax[0], qmax[1]), max(qmax[2], qmax[3]));
            int e2 = 0;
            frexpf(bf16_bits_to_f32(mx), &e2);   // max |q| < 2^e2
            const int sh = e2 > 15 ? e2 - 15 : 0;
            const float qs = ldexpf(1.f, -sh);
            if (tid == 0) *qscale = ldexpf(1.f, sh);
#pragma unroll
            for (int half = 0; half < 2; half++) {
                uint4 u[18];   // 18 loads in flight
#pragma unroll
                for (int c = 0; c < 18; c++)
                    u[c] = *reinterpret_cast<const uint4*>(qrow + 144 * half + 8 * c);
#pragma unroll
                for (int c = 0; c < 18; c++) {
                    const int d0 = 288 * hf + 144 * half + 8 * c;
                    uint32_t w[4] = {u[c].x, u[c].y, u[c].z, u[c].w};
#pragma unroll
                    for (int z = 0; z < 4; z++) {
                        float2 f = bf16x2_to_f32(w[z]);
                        if (d0 >= kD - kRopeDims) {
                            const int pj = (d0 - (kD - kRopeDims)) / 2 + z;
                            f = make_float2(f.x * rqc[pj] - f.y * rqs[pj], f.x * rqs[pj] + f.y * rqc[pj]);
                        }
                        w[z] = pack_f16x2(f.x * qs, f.y * qs);
                    }
                    *cell8(sQ, kQBlk, r, d0) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(qfull);
        }
        // tiles: 4 threads per key row, quarter qt
        const int kr = tid >> 2, qt = tid & 3;
        // the valid keys of a tile: this warp's 8 rows (lanes 0, 4, ..., 28 carry them); then
        // the tile is handed to the MMA issuer
        auto publish = [&](int kb, bool vrow) {
            const uint32_t bal = __ballot_sync(0xffffffffu, vrow && qt == 0);
            uint32_t m8 = 0;
#pragma unroll
            for (int i = 0; i < 8; i++) m8 |= ((bal >> (4 * i)) & 1u) << i;
            if (lane == 0) smask[kb * 4 + warp] = (uint8_t)m8;
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&kfull[kb]);
        };
        // ---- the window tile (global tile `rank`, this rank's first) into key buffer 0 ----
        // (a fresh buffer: no wait).  RMSNorm over all 576 channels (the four quarters of a
        // row meet by shuffle), RoPE at the row's own position on 512..575.
        const bool has_win = nloc > 0 && rank < n_wt;
        if (has_win) {
            uint8_t* tile = sK;
            const int wr = rank * kTK + kr;
            const int64_t p = (int64_t)w0 + wr;
            bool vrow = wr < n_win;
            if (vrow && p < a.raw.first(b, a.seq_len[b])) {
                vrow = false;
                if (qt == 0) flag(a.st, CSA_DEV_OOB);
            }
            const uint16_t* src =
                vrow ? a.kv + a.raw.row(b, p) * (int64_t)kD : nullptr;
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
                sincosf((float)(rank * kTK + er) * rf[pj], &sb_, &cb_);
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
                        w[z] = pack_f16x2(f.x, f.y);
                    }
                    *cl = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            publish(0, vrow);
        }
        // ---- the selected entries ----
        // Each thread converts its quarter of a key row from registers (e4m3 x scale ->
        // fp16, the bf16 RoPE channels to fp16) into the key buffer: the 8 lanes of two
        // rows store to 8 distinct 16-byte columns of the swizzle (no bank conflict).  Two
        // register sets: the loads of tile j + 2 are issued as soon as tile j is converted,
        // so every gather has two tiles' time to arrive.
        // When the rank has entry tiles, the loop starts with two dry steps (j = j0 - 2,
        // j0 - 1), before the wait: they convert zeros through the loop's own code, one per
        // register set, into the spare key buffers 1 and 2 and publish nothing, so that the
        // tiles after the wait do not run from a cold instruction cache (the previous
        // kernels evict the code from L2).  Such a rank writes its partial state over the
        // buffers only after all of its MMAs, hence after the dry steps.
        const int j0 = has_win ? 1 : 0;
        EntryQuarter exa, exb;
#pragma unroll
        for (int u = 0; u < 8; u++) exa.f[u] = exb.f[u] = make_uint4(0u, 0u, 0u, 0u);
        exa.rope[0] = exa.rope[1] = exb.rope[0] = exb.rope[1] = make_uint4(0u, 0u, 0u, 0u);
        exa.sc = exb.sc = make_float4(0.f, 0.f, 0.f, 0.f);
        exa.valid = exb.valid = true;
        auto entry_of = [&](int j) { return (rank + kCl * j - n_wt) * kTK + kr; };
        // converts tile j from `ex`, then issues tile j + 2's loads into it
        auto tile_step = [&](int j, EntryQuarter& ex) -> bool {
            const bool dry = j < j0;
            const int kb = dry ? 1 + ((j - j0) & 1) : j % kKBuf;
            uint8_t* tile = sK + kb * kKBytes;
            // this key buffer is free once the P V of the tile kKBuf back has completed
            if (j >= kKBuf && !mbar_wait_warp(&kfree[kb], ((j / kKBuf) & 1) ^ 1, abort_flag, a.st))
                return false;
            const bool vrow = ex.valid;
            const float scs[4] = {ex.sc.x, ex.sc.y, ex.sc.z, ex.sc.w};
#pragma unroll
            for (int u = 0; u < 8; u++) {
                uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
                if (vrow) dequant16(ex.f[u], pack_f16x2(scs[u >> 1], scs[u >> 1]), lo, hi);
                const int d0 = 64 * u + 16 * qt;
                *cell8(tile, kKBlk, kr, d0) = lo;
                *cell8(tile, kKBlk, kr, d0 + 8) = hi;
            }
            // the RoPE channels are stored as bf16: to fp16 (exact within the fp16 range)
#pragma unroll
            for (int u = 0; u < 2; u++) {
                uint4 h = make_uint4(0u, 0u, 0u, 0u);
                if (vrow) {
                    const uint32_t w[4] = {ex.rope[u].x, ex.rope[u].y, ex.rope[u].z, ex.rope[u].w};
                    uint32_t o[4];
#pragma unroll
                    for (int z = 0; z < 4; z++) {
                        const float2 f = bf16x2_to_f32(w[z]);
                        o[z] = pack_f16x2(f.x, f.y);
                    }
                    h = make_uint4(o[0], o[1], o[2], o[3]);
                }
                *cell8(tile, kKBlk, kr, 512 + 16 * qt + 8 * u) = h;
            }
            if (dry) return true;
            publish(kb, vrow);
            if (j + 2 < nloc) fetch_entry(a, sidx, entry_of(j + 2), n_vis, b, row0, qt, ex);
            return true;
        };
        const int jend = nloc > j0 ? nloc : j0 + 1;   // the wait below runs in every case
        for (int j = nloc > j0 ? j0 - 2 : j0; j < jend && ok; j += 2) {
            if (j == j0) {
                // ---- the index row: the first read of another kernel's output ----
                // Every loader thread waits for the previous grid (the top-k writes the
                // index row, compression the entries), then the row is staged in shared
                // memory.  (Bulk L2 prefetches of the entry rows, one per row through the
                // copy engine, took longer to issue than the gathers they were to speed up.)
                pdl_wait();
                if (tid == 0) pdl_trigger();
                if (valid) {
                    // all of the row's loads in flight at once (16-byte loads when aligned)
                    const int32_t* src = a.idx + (int64_t)qi * a.k;
                    if ((a.k & 3) == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0) {
                        const int n4 = a.k >> 2;   // <= kMaxK / 4 = 4 per thread
                        int4 v[kMaxK / 4 / 128];
#pragma unroll
                        for (int u = 0; u < kMaxK / 4 / 128; u++)
                            if (tid + 128 * u < n4) v[u] = reinterpret_cast<const int4*>(src)[tid + 128 * u];
#pragma unroll
                        for (int u = 0; u < kMaxK / 4 / 128; u++)
                            if (tid + 128 * u < n4) reinterpret_cast<int4*>(sidx)[tid + 128 * u] = v[u];
                    } else {
                        int v[kMaxK / 128];
#pragma unroll
                        for (int u = 0; u < kMaxK / 128; u++)
                            v[u] = tid + 128 * u < a.k ? src[tid + 128 * u] : -1;
#pragma unroll
                        for (int u = 0; u < kMaxK / 128; u++)
                            if (tid + 128 * u < a.k) sidx[tid + 128 * u] = v[u];
                    }
                }
                asm volatile("bar.sync 3, 128;" ::: "memory");
                exa.valid = exb.valid = false;
                if (j0 < nloc) fetch_entry(a, sidx, entry_of(j0), n_vis, b, row0, qt, exa);
                if (j0 + 1 < nloc) fetch_entry(a, sidx, entry_of(j0 + 1), n_vis, b, row0, qt, exb);
            }
            if (j < nloc) ok = tile_step(j, exa);
            if (ok && j + 1 < nloc) ok = tile_step(j + 1, exb);
        }
    } else if (warp == 4 || warp >= kFirstSWarp) {
        if (lane == 0 && nloc > 0) {
            // ---------------- MMA issuers ----------------
            // One tcgen05.mma costs its issuing thread tens of cycles whatever its shape, and
            // S takes 36 per tile: of every tile, warp kFirstSWarp issues the K steps of
            // partials 0 and 2, warp kFirstSWarp + 1 those of partials 1 and 3 (a partial's
            // steps always from one thread, in order), into S buffer j % 2; P V by warp 4.
            // K buffer kb is released by P V's commit: the tile's S was complete before its P
            // (hence its P V) existed.
            bool ok = true;
            if (warp >= kFirstSWarp) {
                const int e = warp - kFirstSWarp;   // partials e and e + 2 of every tile
                ok = mbar_wait(qfull, 0, abort_flag, a.st);
                tc_fence_after();
                for (int j = 0; j < nloc && ok; j++) {
                    const int kb = j % kKBuf, sb = j & 1;
                    if (!mbar_wait(&kfull[kb], (j / kKBuf) & 1, abort_flag, a.st) ||
                        !mbar_wait(&sfree[sb], ((j >> 1) & 1) ^ 1, abort_flag, a.st)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint8_t* tile = sK + kb * kKBytes;
#pragma unroll 1
                    for (int cb = 0; cb < kNB; cb++) {
                        const uint64_t ad = smem_desc_k_sw128(sQ + cb * kQBlk);
                        const uint64_t bd = smem_desc_k_sw128(tile + cb * kKBlk);
#pragma unroll
                        for (int kk = e; kk < 4; kk += 2)   // K = 16 fp16 = 32 bytes, partial kk
                            mma_f16(tmem + s_col(sb, kk), ad + 2 * kk, bd + 2 * kk, kIdescS,
                                    cb ? 1u : 0u);
                    }
                    mma_commit(&sfull[sb]);
                }
            } else {
                for (int j = 0; j < nloc && ok; j++) {
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
            }
            // drain: every issuer's MMAs complete before TMEM is released
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
        // S carries the query's 2^-s scaling: the softmax scale takes 2^s (exact)
        float sl2 = a.scale_log2;
        if (nloc > 0) {
            if (mbar_wait_warp(qfull, 0, abort_flag, a.st)) sl2 *= *qscale;
        }
        bool ok = true;
        for (int j = 0; j < nloc && ok; j++) {
            const int sb = j & 1;
            if (!mbar_wait_warp(&sfull[sb], (j >> 1) & 1, abort_flag, a.st)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // S = (p0 + p2) + (p1 + p3): lanes 0-15 read partials 0 and 2 of head hl, lanes
            // 16-31 partials 1 and 3 of the same head; one exchange across the half-warps
            // gives every lane the same sums (a fixed order, whatever the batch)
            uint32_t sv[kTK];
            {
                uint32_t s0[kTK], s1[kTK];
                tmem_ld32(tmem + s_col(sb, 0) + lane_base, s0);
                tmem_ld32(tmem + s_col(sb, 2) + lane_base, s1);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < kTK; c++) {
                    const float v = __uint_as_float(s0[c]) + __uint_as_float(s1[c]);
                    sv[c] = __float_as_uint(v + __shfl_xor_sync(0xffffffffu, v, 16));
                }
            }
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
            const float tmax = rmax * sl2;
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
                    const float p0 = ex2_approx(fmaf(__uint_as_float(sv[2 * c]), sl2, nm));
                    const float p1 = ex2_approx(fmaf(__uint_as_float(sv[2 * c + 1]), sl2, nm));
                    rs += p0 + p1;
                    pk[c] = pack_f16x2(p0, p1);
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
        if (ntiles > 0 && ok) {
            // ---- this rank's partial state into its own shared memory ----
            // Every MMA of this rank is complete, so Q / K / P may take it.  Lanes 0-15 hold
            // head hl's channels 0-255 (then 512-575), lanes 16-31 its channels 256-511.
            tc_fence_after();
            float* prow = part + hl * kPS;
            const int half = lane >> 4;
#pragma unroll 1
            for (int cc = 0; cc < 5; cc++) {
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
                    float* dst = prow + (cc < 4 ? 256 * half + 64 * cc : 512);
#pragma unroll
                    for (int z = 0; z < 64; z += 4)
                        *reinterpret_cast<float4*>(dst + z) =
                            make_float4(__uint_as_float(ov[z]), __uint_as_float(ov[z + 1]),
                                        __uint_as_float(ov[z + 2]), __uint_as_float(ov[z + 3]));
                }
            }
            if (mine) {
                part[kPartML + hl] = mref;
                part[kPartML + kHC + hl] = lrun;
            }
            tc_fence_before();
            // released to every rank of the cluster
            fence_cluster();
            __syncwarp();
            if (lane == 0)
                for (int rr = 0; rr < kCl; rr++) mbar_arrive_cluster(mapa(cpart_full, (uint32_t)rr));
        }
    }

    // ---- combine: this rank's kHO heads, by the loader and softmax warps (256 threads) ----
    // Each pulls the kCl partial states of its heads from the ranks' shared memory
    // (ld.shared::cluster, 16 consecutive bytes per lane) and sums them in rank order.
    if ((warp < 4 || (warp > 4 && warp < kFirstSWarp)) && ntiles > 0) {
        const int ci = warp < 4 ? threadIdx.x : threadIdx.x - 32;   // 0 .. 255
        const bool okc = mbar_wait_cluster_warp(cpart_full, 0, abort_flag, a.st);
        if (named_barrier_and(2, 256, okc)) {
            // the combine weights, one thread per head, the sink first:
            // M = max(sink, m_r), w_r = 2^(m_r - M), L = 2^(sink - M) + sum_r w_r l_r
            if (ci < kHO) {
                const int h = rank * kHO + ci;
                const float sk = a.sink[kHC * g + h] * kLog2e;
                float mr[kCl], lr[kCl];
#pragma unroll
                for (int rr = 0; rr < kCl; rr++) {
                    mr[rr] = ld_cluster_f32(mapa(part + kPartML + h, (uint32_t)rr));
                    lr[rr] = ld_cluster_f32(mapa(part + kPartML + kHC + h, (uint32_t)rr));
                }
                float M = sk;
#pragma unroll
                for (int rr = 0; rr < kCl; rr++) M = fmaxf(M, mr[rr]);
                float L = (M == -INFINITY || sk == -INFINITY) ? 0.f : exp2f(sk - M);
#pragma unroll
                for (int rr = 0; rr < kCl; rr++) {
                    const float wgt = (mr[rr] == -INFINITY) ? 0.f : exp2f(mr[rr] - M);
                    L = fmaf(wgt, lr[rr], L);
                    swt[ci * kWtStride + rr] = wgt;
                }
                swt[ci * kWtStride + kCl] = L > 0.f ? 1.f / L : 0.f;
            }
            asm volatile("bar.sync 2, 256;" ::: "memory");
            // the output may still be read by the kernel before this one: wait for it
            // (long finished by now whenever this rank gathered entries)
            pdl_wait();
            // (head, 4 channels) per work unit: sum_r w_r O_r / L, inverse RoPE, 4 bf16
#pragma unroll 3
            for (int w = ci; w < kHO * (576 / 4); w += 256) {
                const int lh = w / (576 / 4), c4 = (w - lh * (576 / 4)) * 4;
                const int h = rank * kHO + lh;
                float4 v[kCl];
#pragma unroll
                for (int rr = 0; rr < kCl; rr++) v[rr] = ld_cluster_f4(mapa(part + h * kPS + c4, (uint32_t)rr));
                const float invL = swt[lh * kWtStride + kCl];
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int rr = 0; rr < kCl; rr++) {
                    const float wgt = swt[lh * kWtStride + rr];
                    acc.x = fmaf(wgt, v[rr].x, acc.x);
                    acc.y = fmaf(wgt, v[rr].y, acc.y);
                    acc.z = fmaf(wgt, v[rr].z, acc.z);
                    acc.w = fmaf(wgt, v[rr].w, acc.w);
                }
                acc = make_float4(acc.x * invL, acc.y * invL, acc.z * invL, acc.w * invL);
                if (c4 >= kD - kRopeDims) {
                    // rotation by -t: (x, y) -> (x cos + y sin, y cos - x sin)
                    const int pj = (c4 - (kD - kRopeDims)) >> 1;
                    const float c0 = rqc[pj], s0 = rqs[pj], c1 = rqc[pj + 1], s1 = rqs[pj + 1];
                    acc = make_float4(acc.x * c0 + acc.y * s0, acc.y * c0 - acc.x * s0,
                                      acc.z * c1 + acc.w * s1, acc.w * c1 - acc.z * s1);
                }
                *reinterpret_cast<uint2*>(a.out + ((int64_t)qi * a.H + kHC * g + h) * kD + c4) =
                    make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
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
    a.er = aa.er;
    a.kv = aa.kv;
    a.raw = aa.raw;
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
