// Steps a1/a2: CSA (m=4, 8 pooled tokens) and HCA (m'=128, 128 pooled tokens) compression.
//
// "DeepSeek-V4 深度分析报告" 2.1: CSA turns every 4 tokens into one entry drawing on 8
// tokens (its block and the previous one); HCA turns every 128 tokens into one entry.
// Per channel: softmax over the pooled tokens of (gate logit + positional bias row),
// weighted sum of the raw KV, then RMSNorm over the head dim and RoPE on the last 64
// channels at the block-end position, then bf16 or fp8(1x128)+bf16 storage.
//
// One CTA per entry; each thread owns 4 consecutive channels (8-byte bf16x4 loads, so a
// warp reads 256 contiguous bytes of a token row).  The softmax runs online over the
// pooled tokens in fp32; RMSNorm reduces over the CTA; the RoPE pairs of a thread's 4
// channels are local to it.  HBM-bound: every raw token row is read once per entry that
// pools it (twice for CSA's overlap; the second read mostly hits L2).
#include "launchers.cuh"

namespace csa {

// Tokens of one entry are split over TG token groups (along the token axis) that walk
// chunks of 8 tokens; a thread loads a chunk's 8 tokens x 4 channels at once (and the next
// chunk's before reducing the current one), keeps an online softmax state per channel, and
// the token groups merge their states pairwise in a fixed tree through shared memory.  All
// inputs (item lists, offsets, raw tokens, the positional bias) are read before the wait on
// the previous kernel: no earlier libcsa kernel writes them, so in a PDL pipeline their
// latency overlaps it; only the entry store needs the wait.
constexpr int kChunkTok = 8;
constexpr int kMaxMergeSlots = 640;   // TG * channel lanes

struct Chunk {
    uint2 z[kChunkTok], v[kChunkTok];
};

__device__ __forceinline__ void load_chunk(const uint16_t* __restrict__ kv,
                                           const uint16_t* __restrict__ gate, const RawRows& raw,
                                           int b, int64_t first_pos, int D, int c0, Chunk& ch) {
    // positions before the sequence start (entry 0 of CSA) re-read position 0's row and
    // are masked out of the softmax by the caller
#pragma unroll
    for (int jj = 0; jj < kChunkTok; jj++) {
        const int64_t p = first_pos + jj;
        const int64_t row = raw.row(b, p >= 0 ? p : 0);
        ch.z[jj] = *reinterpret_cast<const uint2*>(gate + row * D + c0);
        ch.v[jj] = *reinterpret_cast<const uint2*>(kv + row * D + c0);
    }
}

// NCH: chunks per token group (1 for CSA's 8 tokens, and for HCA's 128 tokens over 16
// token groups; 4 for HCA over 4 token groups).  With one chunk the bias rows of the chunk
// sit in registers next to its tokens; with several the next chunk's tokens do, and the
// bias is read where it is used.
template <int SPAN, int NCH>
__global__ void __launch_bounds__(SPAN == 8 ? 160 : (NCH == 1 ? 512 : 640)) compress_kernel(
    const uint16_t* __restrict__ kv, const uint16_t* __restrict__ gate,
    const float* __restrict__ bias, const int64_t* __restrict__ seq_len, const RawRows raw,
    const EntryRows er, const int32_t* __restrict__ item_seq, const int32_t* __restrict__ item_ent, int B, int m,
    int D, int fmt, double log2_theta, float eps, uint8_t* __restrict__ entries,
    int32_t* __restrict__ dev_status) {
    __shared__ float red[8];
    __shared__ float4 st_m[SPAN == 8 ? 1 : kMaxMergeSlots], st_d[SPAN == 8 ? 1 : kMaxMergeSlots],
        st_a[SPAN == 8 ? 1 : kMaxMergeSlots];
    const int64_t it = blockIdx.x;
    const int b = item_seq[it];
    const int64_t i = item_ent[it];
    bool ok = !(b < 0 || b >= B || i < 0);
    const int64_t first = (i + 1) * (int64_t)m - SPAN;
    const int64_t pos0 = ok ? raw.first(b, seq_len[b]) : 0;
    const int64_t erow = ok ? er.row(b, i) : 0;
    // every pooled token must be stored: positions max(first, 0) .. (i+1)m-1
    if (ok && ((first > 0 ? first : 0) < pos0 || (i + 1) * (int64_t)m > seq_len[b])) ok = false;
    const int cw = 32 * ((D / 4 + 31) / 32);     // channel lanes per token group
    const int TG = blockDim.x / cw;               // token groups
    constexpr int nch = NCH;                      // chunks per token group
    const int tid = threadIdx.x;
    const int cl = tid % cw, tg = tid / cw;
    const int c0 = cl * 4;
    const bool active = ok && c0 < D;

    float mx[4], den[4], acc[4];
#pragma unroll
    for (int u = 0; u < 4; u++) {
        mx[u] = -INFINITY;
        den[u] = 0.f;
        acc[u] = 0.f;
    }
    const int j_begin = tg * nch * kChunkTok;
    Chunk cur, nxt;
    float4 bcur[NCH == 1 ? kChunkTok : 1] = {};   // the chunk's positional bias rows (one chunk)
    auto bias_row = [&](int j) -> float4 {
        if constexpr (NCH == 1) return bcur[j - j_begin];
        else return *reinterpret_cast<const float4*>(bias + (int64_t)j * D + c0);
    };
    if (active) {
        load_chunk(kv, gate, raw, b, first + j_begin, D, c0, cur);
        if constexpr (NCH == 1) {
#pragma unroll
            for (int jj = 0; jj < kChunkTok; jj++)
                bcur[jj] = *reinterpret_cast<const float4*>(bias + (int64_t)(j_begin + jj) * D + c0);
        }
    }
    pdl_wait();   // entries may still be read by the previous step's attention
    pdl_trigger();
    if (!ok) {
        if (threadIdx.x == 0) flag(dev_status, CSA_DEV_OOB);
        return;
    }
    if (active) {
#pragma unroll 1
        for (int c = 0; c < nch; c++) {
            const int j0 = j_begin + c * kChunkTok;
            if (c + 1 < nch) load_chunk(kv, gate, raw, b, first + j0 + kChunkTok, D, c0, nxt);
            float cm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int jj = 0; jj < kChunkTok; jj++) {
                if (first + j0 + jj < 0) continue;
                const float4 bb = bias_row(j0 + jj);
                const float2 z01 = bf16x2_to_f32(cur.z[jj].x), z23 = bf16x2_to_f32(cur.z[jj].y);
                cm[0] = fmaxf(cm[0], z01.x + bb.x);
                cm[1] = fmaxf(cm[1], z01.y + bb.y);
                cm[2] = fmaxf(cm[2], z23.x + bb.z);
                cm[3] = fmaxf(cm[3], z23.y + bb.w);
            }
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const float M = fmaxf(mx[u], cm[u]);
                if (M != -INFINITY && mx[u] != -INFINITY) {
                    const float sc = expf(mx[u] - M);
                    den[u] *= sc;
                    acc[u] *= sc;
                }
                mx[u] = M;
            }
#pragma unroll
            for (int jj = 0; jj < kChunkTok; jj++) {
                if (first + j0 + jj < 0) continue;
                const float4 bb = bias_row(j0 + jj);
                const float2 z01 = bf16x2_to_f32(cur.z[jj].x), z23 = bf16x2_to_f32(cur.z[jj].y);
                const float2 v01 = bf16x2_to_f32(cur.v[jj].x), v23 = bf16x2_to_f32(cur.v[jj].y);
                const float l[4] = {z01.x + bb.x, z01.y + bb.y, z23.x + bb.z, z23.y + bb.w};
                const float v[4] = {v01.x, v01.y, v23.x, v23.y};
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const float p = expf(l[u] - mx[u]);
                    den[u] += p;
                    acc[u] = fmaf(p, v[u], acc[u]);
                }
            }
            if (c + 1 < nch) cur = nxt;
        }
    }
    if (TG > 1) {
        // merge the token groups' states pairwise: (0,1) (2,3) .., then (0,2) .., a fixed
        // tree; a group's state goes to its own slot, its partner reads it
        for (int stride = 1; stride < TG; stride <<= 1) {
            if (tg % (2 * stride) == stride) {
                const int slot = tg * cw + cl;
                st_m[slot] = make_float4(mx[0], mx[1], mx[2], mx[3]);
                st_d[slot] = make_float4(den[0], den[1], den[2], den[3]);
                st_a[slot] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            }
            __syncthreads();
            if (tg % (2 * stride) == 0 && tg + stride < TG) {
                const int slot = (tg + stride) * cw + cl;
                const float4 gm = st_m[slot], gd = st_d[slot], ga = st_a[slot];
                const float om[4] = {gm.x, gm.y, gm.z, gm.w}, od[4] = {gd.x, gd.y, gd.z, gd.w},
                            oa[4] = {ga.x, ga.y, ga.z, ga.w};
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const float M = fmaxf(mx[u], om[u]);
                    if (M == -INFINITY) continue;
                    const float s0 = mx[u] == -INFINITY ? 0.f : expf(mx[u] - M);
                    const float s1 = om[u] == -INFINITY ? 0.f : expf(om[u] - M);
                    den[u] = den[u] * s0 + od[u] * s1;
                    acc[u] = acc[u] * s0 + oa[u] * s1;
                    mx[u] = M;
                }
            }
        }
        if (tg > 0) return;
    }
    float e[4] = {0.f, 0.f, 0.f, 0.f};
    if (active) {
#pragma unroll
        for (int u = 0; u < 4; u++) e[u] = acc[u] / den[u];
    }

    // RMSNorm over all D channels (unit weight); threads of token group 0 only from here.
    float ss = e[0] * e[0] + e[1] * e[1] + e[2] * e[2] + e[3] * e[3];
    ss = warp_sum(ss);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    if (blockDim.x > cw) {
        asm volatile("bar.sync 1, %0;" ::"r"(cw) : "memory");
    } else {
        __syncthreads();
    }
    float tot = 0.f;
    for (int w = 0; w < cw / 32; w++) tot += red[w];
    const float r = rsqrtf(tot / (float)D + eps);
#pragma unroll
    for (int u = 0; u < 4; u++) e[u] *= r;

    // RoPE on the last 64 channels at the block-end position.
    if (active && c0 >= D - kRopeDims) {
        const double pos = (double)((i + 1) * (int64_t)m - 1);
        const int pair = (c0 - (D - kRopeDims)) >> 1;
#pragma unroll
        for (int u = 0; u < 2; u++) {
            float cs, sn;
            rope_cos_sin(pos, pair + u, log2_theta, cs, sn);
            const float x = e[2 * u], y = e[2 * u + 1];
            e[2 * u] = x * cs - y * sn;
            e[2 * u + 1] = x * sn + y * cs;
        }
    }

    // Store.
    if (fmt == CSA_KV_BF16) {
        if (active) {
            uint8_t* dst = entries + erow * (int64_t)(2 * D) + 2 * c0;
            *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(e[0], e[1]), pack_bf16x2(e[2], e[3]));
        }
    } else {  // CSA_KV_FP8_576: warps 0..3 hold channels 0..511 (one 1x128 block per warp)
        uint8_t* dst = entries + erow * 656;
        const int warp = tid >> 5, lane = tid & 31;
        if (warp < 4) {
            float amax = fmaxf(fmaxf(fabsf(e[0]), fabsf(e[1])), fmaxf(fabsf(e[2]), fabsf(e[3])));
            amax = warp_max(amax);
            float scale = amax / 448.0f;
            if (!(scale > 0.f)) scale = 1.f;
            uint32_t codes = 0;
#pragma unroll
            for (int u = 0; u < 4; u++) codes |= f32_to_e4m3_satfinite(e[u] / scale) << (8 * u);
            *reinterpret_cast<uint32_t*>(dst + c0) = codes;
            if (lane == 0) *reinterpret_cast<float*>(dst + 512 + 4 * warp) = scale;
        } else if (active) {
            *reinterpret_cast<uint2*>(dst + 528 + 2 * (c0 - 512)) =
                make_uint2(pack_bf16x2(e[0], e[1]), pack_bf16x2(e[2], e[3]));
        }
    }
}

cudaError_t launch_compress(int span, const void* kv, const void* gate, const float* bias,
                            const int64_t* seq_len, const RawRows& raw, const EntryRows& er,
                            const int32_t* item_seq, const int32_t* item_ent, int64_t n_items,
                            int B, int m, int D, int fmt, float theta, float eps, void* entries,
                            int32_t* st, cudaStream_t stream) {
    if (n_items == 0) return cudaSuccess;
    const int cw = 32 * ((D / 4 + 31) / 32);        // channel lanes: 32 (D=128) or 160 (576)
    const double log2_theta = log2((double)theta);
    const dim3 grid((unsigned)n_items);
    LaunchScope scope(kKCompress, stream);
    if (span == 8) {
        return launch_pdl(compress_kernel<8, 1>, grid, dim3(cw), 0, stream, (const uint16_t*)kv,
                          (const uint16_t*)gate, bias, seq_len, raw, er, item_seq, item_ent, B,
                          m, D, fmt, log2_theta, eps, (uint8_t*)entries, st);
    } else {
        // token groups: 16 x 8 tokens (D=128) or 4 x 32 tokens (D=576)
        if (cw == 32)
            return launch_pdl(compress_kernel<128, 1>, grid, dim3(16 * cw), 0, stream,
                              (const uint16_t*)kv, (const uint16_t*)gate, bias, seq_len, raw, er,
                              item_seq, item_ent, B, m, D, fmt, log2_theta, eps,
                              (uint8_t*)entries, st);
        return launch_pdl(compress_kernel<128, 4>, grid, dim3(4 * cw), 0, stream,
                          (const uint16_t*)kv, (const uint16_t*)gate, bias, seq_len, raw, er,
                          item_seq, item_ent, B, m, D, fmt, log2_theta, eps, (uint8_t*)entries,
                          st);
    }
    return cudaGetLastError();
}

}  // namespace csa
