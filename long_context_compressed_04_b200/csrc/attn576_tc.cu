// Step a5 on the 5th-generation tensor cores for 576-dim compressed entries stored as
// 512 FP8 E4M3 channels (one fp32 scale per 128) + 64 BF16 RoPE channels (656-byte rows),
// with 64 or more query heads: shared-KV MQA over the selected entries plus the sliding
// window, with the attention sink and partial / inverse RoPE ("DeepSeek-V4 深度分析报告"
// 2.1 CSA and "其他注意力技术细节").
//
// One CTA per (query, group of 64 heads).  The keys of the query are tiles of 64: the
// window's raw rows first (RMSNormed and RoPEd here), then the selected entries.
//   warps 0-3  loaders: the query's 64 head rows RoPEd at t into shared memory once; per
//              tile, 2 threads per key row dequantize the gathered FP8 row (or normalise the
//              raw window row) into bf16, 128-byte swizzled, 9 blocks of 64 channels; the
//              next entry tile's rows are copied (cp.async) into a raw staging buffer while
//              the previous tile is still in use.
//   warp 4     TMEM allocation; lane 0 issues tcgen05.mma kind::f16:
//              S = Q K^T (M = 64 heads, N = 64 keys, 36 K steps of 16 channels) into one of
//              two S buffers, then O += P V straight into the TMEM accumulator: channels
//              0-255 in TMEM lanes 0-15 of each quarter, 256-511 in lanes 16-31, 512-575 in
//              lanes 0-15 again (N = 256 + 256 + 64), V being the key tile read MN-major.
//   warps 5-8  online softmax in the log2 domain, one head row per lane: P as bf16 into
//              shared memory; the running maximum is a reference that moves only when a
//              tile's maximum exceeds it by 2^8, and then the head's O row in TMEM is
//              rescaled; finally the sink, the normalisation, inverse RoPE and the store.
// A 64 x 576 fp32 accumulator takes 320 TMEM columns, and the query's Q tile (72 KB) and
// one key tile (72 KB) fill most of shared memory: hence 64 heads per CTA, 64-key tiles.
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
constexpr int kTK = 64;                  // keys per tile (MMA N of S)
constexpr int kBlk = 64 * 128;           // one 64-row x 128-byte swizzled block
constexpr int kQBytes = kNB * kBlk;      // 72 KB
constexpr int kKBytes = kNB * kBlk;      // 72 KB
constexpr int kPBytes = kBlk;            // 8 KB
constexpr int kRowBytes = 656;
constexpr int kThreads = 288;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.f;          // the reference maximum moves by more than 2^8 only
constexpr uint32_t kColO = 0;            // O channels 0-255 (lanes 0-15) / 256-511 (lanes 16-31)
constexpr uint32_t kColOr = 256;         // O channels 512-575 (lanes 0-15)
constexpr uint32_t kColS = 320;          // S buffers at 320 and 384 (lanes 0-15)
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxK = 2048;

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
// [9 blocks][64 rows x 128 B] swizzled tile.
__device__ __forceinline__ void put8(uint8_t* tile, int r, int d0, uint4 v) {
    *reinterpret_cast<uint4*>(tile + (d0 >> 6) * kBlk + swz(r, (d0 & 63) >> 3)) = v;
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

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sm100::smem_addr(dst)),
                 "l"(src)
                 : "memory");
}

// Starts copying one loader thread's half of entry v of the query's index row (staged in
// shared memory) into its raw row slot: fp8 channels [256 hf, 256 hf + 256), RoPE channels
// [32 hf, 32 hf + 32), and (hf = 0) the four scales.  False for an invalid index (an
// out-of-range one is flagged once per row).
__device__ __forceinline__ bool fetch_entry(const A576Args& a, const int32_t* sidx, int v,
                                            int n_vis, int64_t row0, int hf, uint8_t* raw) {
    const int e = v < a.k ? sidx[v] : -1;
    bool valid = false;
    if (e >= 0) {
        if (e < n_vis && row0 + e < a.ent_rows) {
            valid = true;
        } else if (hf == 0) {
            flag(a.st, CSA_DEV_OOB);
        }
    }
    if (valid) {
        const uint8_t* er = a.entries + (row0 + e) * (int64_t)kRowBytes;
#pragma unroll
        for (int u = 0; u < 16; u++) cp_async16(raw + 256 * hf + 16 * u, er + 256 * hf + 16 * u);
#pragma unroll
        for (int u = 0; u < 4; u++)
            cp_async16(raw + 528 + 64 * hf + 16 * u, er + 528 + 64 * hf + 16 * u);
        if (hf == 0) cp_async16(raw + 512, er + 512);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    return valid;
}

__global__ void __launch_bounds__(kThreads, 1) attn576_tc_kernel(const A576Args a) {
    using namespace sm100;
    constexpr uint32_t kIdescS = instr_desc(1, 1, 64, 64);
    constexpr uint32_t kIdescPV = instr_desc(1, 1, 64, 256, 1);
    constexpr uint32_t kIdescPVr = instr_desc(1, 1, 64, 64, 1);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* sQ = smem;                                   // [9][64 x 128 B]
    uint8_t* sK = sQ + kQBytes;                           // [9][64 x 128 B]
    uint8_t* sP = sK + kKBytes;                           // [2][64 x 128 B]
    uint16_t* smask = reinterpret_cast<uint16_t*>(sP + 2 * kPBytes);   // [2][4] valid keys
    float* rqc = reinterpret_cast<float*>(smask + 8);     // [32] cos / sin of pair j at t
    float* rqs = rqc + 32;
    float* rf = rqs + 32;                                 // [32] frequency of pair j
    float* rwc = rf + 32;                                 // [32] cos / sin of pair j at w0
    float* rws = rwc + 32;
    int32_t* sidx = reinterpret_cast<int32_t*>(rws + 32); // [kMaxK] the query's index row
    uint8_t* sRaw = reinterpret_cast<uint8_t*>(sidx + kMaxK);   // [64][656] next entry rows
    uint64_t* bars = reinterpret_cast<uint64_t*>(sRaw + kTK * kRowBytes);
    uint64_t* qfull = bars;          // 4 loader warps
    uint64_t* kfull = bars + 1;      // 4 loader warps
    uint64_t* kfree = bars + 2;      // MMA commit after the tile's P V
    uint64_t* sfull = bars + 3;      // [2] MMA commit
    uint64_t* sfree = bars + 5;      // [2] 4 softmax warps
    uint64_t* pfull = bars + 7;      // [2] 4 softmax warps
    uint64_t* pfree = bars + 9;      // [2] MMA commit
    uint64_t* pvdone = bars + 11;    // MMA commit after every P V
    uint64_t* drain = bars + 12;
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(bars + 13);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_smem + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.H / kHC;
    const int qi = blockIdx.x / G, g = blockIdx.x - qi * G;
    // the query (the same decision in every thread)
    const int b = a.q_seq[qi];
    const int t = a.q_pos[qi];
    const bool valid = b >= 0 && b < a.B && t >= 0 && (int64_t)t < a.seq_len[b];
    if (threadIdx.x == 0) {
        mbar_init(qfull, 4);
        mbar_init(kfull, 4);
        mbar_init(kfree, 1);
        for (int i = 0; i < 2; i++) {
            mbar_init(&sfull[i], 1);
            mbar_init(&sfree[i], 4);
            mbar_init(&pfull[i], 4);
            mbar_init(&pfree[i], 1);
        }
        mbar_init(pvdone, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        mbar_fence_init();
        if (!valid && g == 0) flag(a.st, CSA_DEV_OOB);
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
    tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;

    const int n_vis = valid ? (t + 1) / a.m : 0;
    const int64_t row0 = valid ? a.ent_off[b] : 0;
    const int w0 = t - a.W + 1 > 0 ? t - a.W + 1 : 0;
    const int n_win = a.W > 0 ? t - w0 + 1 : 0;
    const int n_wt = (a.W + kTK - 1) / kTK;          // window tiles (masked past n_win)
    const int n_et = (a.k + kTK - 1) / kTK;          // selected-entry tiles
    const int ntiles = valid ? n_wt + n_et : 0;

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
                    put8(sQ, r, d0, u[c]);
                }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(qfull);
        }
        uint8_t* myraw = sRaw + r * kRowBytes;
        bool ex_valid = false;
        if (n_wt == 0 && ntiles > 0) ex_valid = fetch_entry(a, sidx, r, n_vis, row0, hf, myraw);
        for (int j = 0; j < ntiles && ok; j++) {
            // the key buffer is free once the previous tile's P V has completed
            if (j > 0 && !mbar_wait_warp(kfree, (j - 1) & 1, abort_flag, a.st)) {
                ok = false;
                break;
            }
            bool vrow;
            if (j < n_wt) {
                // window row: RMSNorm over all 576 channels (the two halves meet by shuffle),
                // RoPE at its own position on 512..575
                const int wr = j * kTK + r;
                const int64_t p = (int64_t)w0 + wr;
                vrow = wr < n_win;
                if (vrow && p < a.kv_pos0[b]) {
                    vrow = false;
                    if (hf == 0) flag(a.st, CSA_DEV_OOB);
                }
                const uint16_t* src =
                    vrow ? a.kv + (a.kv_off[b] + p - a.kv_pos0[b]) * (int64_t)kD : nullptr;
                // pass 1: the raw row into the tile (18 loads in flight) and its sum of squares
                float ss = 0.f;
#pragma unroll
                for (int half = 0; half < 2; half++) {
                    uint4 u[18];
#pragma unroll
                    for (int c = 0; c < 18; c++)
                        u[c] = vrow ? *reinterpret_cast<const uint4*>(src + 288 * hf + 144 * half + 8 * c)
                                    : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int c = 0; c < 18; c++) {
                        const uint32_t w[4] = {u[c].x, u[c].y, u[c].z, u[c].w};
#pragma unroll
                        for (int z = 0; z < 4; z++) {
                            const float2 f = bf16x2_to_f32(w[z]);
                            ss += f.x * f.x + f.y * f.y;
                        }
                        put8(sK, r, 288 * hf + 144 * half + 8 * c, u[c]);
                    }
                }
                ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                const float rn = rsqrtf(ss / (float)kD + a.eps);
                // pass 2, in place in shared memory: normalise, RoPE at the row's position
                if (vrow) {
#pragma unroll 4
                    for (int c = 0; c < 36; c++) {
                        const int d0 = 288 * hf + 8 * c;
                        uint4* cell = reinterpret_cast<uint4*>(sK + (d0 >> 6) * kBlk + swz(r, (d0 & 63) >> 3));
                        const uint4 u = *cell;
                        const uint32_t wi[4] = {u.x, u.y, u.z, u.w};
                        uint32_t w[4];
#pragma unroll
                        for (int z = 0; z < 4; z++) {
                            float2 f = bf16x2_to_f32(wi[z]);
                            f.x *= rn;
                            f.y *= rn;
                            if (d0 >= kD - kRopeDims) {
                                // angle (w0 + wr) f_j = w0 f_j (fp64 table) + wr f_j (< 128 rad,
                                // sincosf), combined by the addition formula
                                const int pj = (d0 - (kD - kRopeDims)) / 2 + z;
                                float sb_, cb_;
                                sincosf((float)wr * rf[pj], &sb_, &cb_);
                                const float cs = rwc[pj] * cb_ - rws[pj] * sb_;
                                const float sn = rws[pj] * cb_ + rwc[pj] * sb_;
                                f = make_float2(f.x * cs - f.y * sn, f.x * sn + f.y * cs);
                            }
                            w[z] = pack_bf16x2(f.x, f.y);
                        }
                        *cell = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            } else {
                vrow = ex_valid;
                // this thread's copies, then its partner's (the scales) are visible
                asm volatile("cp.async.wait_group 0;" ::: "memory");
                __syncwarp();
                const float* scl = reinterpret_cast<const float*>(myraw + 512);
                const float sc0 = vrow ? scl[2 * hf] : 0.f, sc1 = vrow ? scl[2 * hf + 1] : 0.f;
#pragma unroll 4
                for (int u = 0; u < 16; u++) {
                    uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
                    if (vrow)
                        dequant16(*reinterpret_cast<const uint4*>(myraw + 256 * hf + 16 * u),
                                  u < 8 ? sc0 : sc1, lo, hi);
                    const int d0 = 256 * hf + 16 * u;
                    put8(sK, r, d0, lo);
                    put8(sK, r, d0 + 8, hi);
                }
#pragma unroll
                for (int u = 0; u < 4; u++)
                    put8(sK, r, 512 + 32 * hf + 8 * u,
                         vrow ? *reinterpret_cast<const uint4*>(myraw + 528 + 64 * hf + 16 * u)
                              : make_uint4(0u, 0u, 0u, 0u));
                // the raw slot is read: the partner may overwrite its half with the next row
                __syncwarp();
            }
            // valid keys of the tile: this warp's 16 rows (even lanes carry them)
            const uint32_t bal = __ballot_sync(0xffffffffu, vrow && hf == 0);
            uint32_t m16 = 0;
#pragma unroll
            for (int i = 0; i < 16; i++) m16 |= ((bal >> (2 * i)) & 1u) << i;
            if (lane == 0) smask[(j & 1) * 4 + warp] = (uint16_t)m16;
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(kfull);
            // the next entry tile's bytes in flight while this one is used
            if (j + 1 >= n_wt && j + 1 < ntiles)
                ex_valid = fetch_entry(a, sidx, (j + 1 - n_wt) * kTK + r, n_vis, row0, hf, myraw);
        }
    } else if (warp == 4) {
        if (lane == 0 && ntiles > 0) {
            // ---------------- MMA issuer ----------------
            bool ok = mbar_wait(qfull, 0, abort_flag, a.st);
            tc_fence_after();
            for (int j = 0; j < ntiles && ok; j++) {
                const int sb = j & 1;
                if (!mbar_wait(kfull, j & 1, abort_flag, a.st) ||
                    !mbar_wait(&sfree[sb], ((j >> 1) & 1) ^ 1, abort_flag, a.st)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t ds = tmem + kColS + (uint32_t)(sb * 64);
#pragma unroll 1
                for (int kb = 0; kb < kNB; kb++) {
                    const uint64_t ad = smem_desc_k_sw128(sQ + kb * kBlk);
                    const uint64_t bd = smem_desc_k_sw128(sK + kb * kBlk);
#pragma unroll
                    for (int kk = 0; kk < 4; kk++)   // K = 16 bf16 = 32 bytes per MMA
                        mma_f16(ds, ad + 2 * kk, bd + 2 * kk, kIdescS, (kb | kk) ? 1u : 0u);
                }
                mma_commit(&sfull[sb]);
                if (!mbar_wait(&pfull[sb], (j >> 1) & 1, abort_flag, a.st)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t pa = smem_desc_k_sw128(sP + sb * kPBytes);
#pragma unroll
                for (int kk = 0; kk < 4; kk++) {   // 16 keys per MMA
                    const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
                    mma_f16(tmem + kColO, pa + 2 * kk, desc_mn(sK + kk * 2048, kBlk), kIdescPV, acc);
                    mma_f16(tmem + kColO + (16u << 16), pa + 2 * kk,
                            desc_mn(sK + 4 * kBlk + kk * 2048, kBlk), kIdescPV, acc);
                    mma_f16(tmem + kColOr, pa + 2 * kk, desc_mn(sK + 8 * kBlk + kk * 2048, kBlk),
                            kIdescPVr, acc);
                }
                mma_commit(kfree);
                mma_commit(&pfree[sb]);
                mma_commit(pvdone);
            }
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
        for (int j = 0; j < ntiles && ok; j++) {
            const int sb = j & 1;
            if (!mbar_wait_warp(&sfull[sb], (j >> 1) & 1, abort_flag, a.st)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sv[64];
            tmem_ld64(tmem + kColS + (uint32_t)(sb * 64) + lane_base, sv);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sfree[sb]);
            const uint16_t* mk = smask + sb * 4;
            const uint32_t mlo = (uint32_t)mk[0] | ((uint32_t)mk[1] << 16);
            const uint32_t mhi = (uint32_t)mk[2] | ((uint32_t)mk[3] << 16);
            float tmax = -INFINITY;
#pragma unroll
            for (int c = 0; c < 64; c++) {
                const bool on = mine && (((c < 32 ? mlo >> c : mhi >> (c - 32)) & 1u) != 0);
                const float xv = on ? __uint_as_float(sv[c]) * a.scale_log2 : -INFINITY;
                sv[c] = __float_as_uint(xv);
                tmax = fmaxf(tmax, xv);
            }
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
            float rs = 0.f;
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < 32; c++) {
                const float x0 = __uint_as_float(sv[2 * c]), x1 = __uint_as_float(sv[2 * c + 1]);
                const float p0 = x0 == -INFINITY ? 0.f : exp2f(x0 - mref);
                const float p1 = x1 == -INFINITY ? 0.f : exp2f(x1 - mref);
                rs += p0 + p1;
                pk[c] = pack_bf16x2(p0, p1);
            }
            lrun += rs;
            if (!mbar_wait_warp(&pfree[sb], ((j >> 1) & 1) ^ 1, abort_flag, a.st)) {
                ok = false;
                break;
            }
            if (mine) {
                uint8_t* prow = sP + sb * kPBytes;
#pragma unroll
                for (int c = 0; c < 8; c++)
                    *reinterpret_cast<uint4*>(prow + swz(hl, c)) =
                        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pfull[sb]);
        }
        if (ok && ntiles > 0) ok = mbar_wait_warp(pvdone, (ntiles - 1) & 1, abort_flag, a.st);
        if (ok && ntiles > 0) {
            tc_fence_after();
            // o = O 2^(mref - M) / (2^(sink - M) + l 2^(mref - M)),  M = max(mref, sink)
            const int h = kHC * g + hl;
            const float sk = a.sink[h] * kLog2e;
            const float M = fmaxf(mref, sk);
            float inv = 0.f;
            if (M != -INFINITY) {
                const float so = mref == -INFINITY ? 0.f : exp2f(mref - M);
                const float L = lrun * so + (sk == -INFINITY ? 0.f : exp2f(sk - M));
                inv = L > 0.f ? so / L : 0.f;
            }
            inv = __shfl_sync(0xffffffffu, inv, lane & 15);
            uint16_t* orow = a.out + ((int64_t)qi * a.H + h) * kD;
            // channels 0-255 (lanes 0-15) and 256-511 (lanes 16-31)
#pragma unroll 1
            for (int cc = 0; cc < 16; cc++) {
                uint32_t ov[16];
                tmem_ld16(tmem + kColO + 16u * cc + lane_base, ov);
                tmem_ld_wait();
                uint32_t w[8];
#pragma unroll
                for (int z = 0; z < 8; z++)
                    w[z] = pack_bf16x2(__uint_as_float(ov[2 * z]) * inv, __uint_as_float(ov[2 * z + 1]) * inv);
                uint4* dst = reinterpret_cast<uint4*>(orow + (mine ? 0 : 256) + 16 * cc);
                dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
            }
            // channels 512-575 (lanes 0-15): inverse RoPE (rotation by -t)
#pragma unroll 1
            for (int cc = 0; cc < 4; cc++) {
                uint32_t ov[16];
                tmem_ld16(tmem + kColOr + 16u * cc + lane_base, ov);
                tmem_ld_wait();
                if (mine) {
                    uint32_t w[8];
#pragma unroll
                    for (int z = 0; z < 8; z++) {
                        const int pj = 8 * cc + z;
                        const float x = __uint_as_float(ov[2 * z]) * inv;
                        const float y = __uint_as_float(ov[2 * z + 1]) * inv;
                        w[z] = pack_bf16x2(x * rqc[pj] + y * rqs[pj], y * rqc[pj] - x * rqs[pj]);
                    }
                    uint4* dst = reinterpret_cast<uint4*>(orow + 512 + 16 * cc);
                    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                }
            }
            tc_fence_before();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

constexpr size_t kSmemBytes = 1024 + kQBytes + kKBytes + 2 * kPBytes + 8 * 2 + 5 * 32 * 4 +
                              kMaxK * 4 + kTK * kRowBytes + 13 * 8 + 16;
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
    return launch_pdl(attn576_tc_kernel, dim3(Q * (aa.H / kHC)), dim3(kThreads), kSmemBytes,
                      stream, a);
}

}  // namespace csa
