// Steps a5/a6 (CUDA-core path): shared-KV MQA over compressed entries plus the sliding
// window, with an attention sink and partial / inverse RoPE.
//
// "DeepSeek-V4 深度分析报告" 2.1 (CSA attends to the top-k entries, HCA to all entries,
// both with a 128-token window branch) and "其他注意力技术细节" (Shared Key-Value MQA:
// every entry is key and value for all heads; Partial RoPE on the last 64 dims with
// inverse RoPE on the output; Attention Sink: a learnable per-head logit, so weights can
// sum to less than 1).
//
// One CTA per (query, group of 16 heads).  The key list is the selected (or all visible)
// entries in the given order, then the window rows in ascending position.  Keys stream
// through shared memory in tiles of 32 rows converted to fp32 (window rows are RMSNormed
// and RoPEd while loading); logits, the online softmax (the sink enters as the initial
// running max with weight 1 and a zero value) and the P.V update run in fp32.  The tile
// order and all reductions are fixed by the query alone: batch-invariant.
#include "launchers.cuh"

namespace csa {

constexpr int kHG = 16;  // heads per CTA
constexpr int kTK = 32;  // keys per tile

// Loads key `vk` of the query's key list as fp32 into row[0..D) (stride 1).  Returns
// whether the key is valid.  One warp per key; lane handles channel pairs lane + 32u.
template <int D>
__device__ __forceinline__ bool load_key(const AttnArgs& a, int b, int t, int n_vis,
                                         int n_sel, int w0, int vk, float* row, int lane) {
    constexpr int NP = D / 64;  // channel pairs per lane
    bool valid = true;
    const uint8_t* erow = nullptr;
    const uint16_t* wrow = nullptr;
    int64_t wpos = 0;
    if (vk < n_sel) {
        const int e = a.idx ? a.idx[(int64_t)blockIdx.y * a.k + vk] : vk;
        if (e < 0) {
            valid = false;
        } else {
            const int64_t re = e < n_vis ? a.er.row(b, e) : -1;
            if (re < 0 || re >= a.ent_rows) {
                valid = false;
                if (lane == 0 && blockIdx.x == 0) flag(a.st, CSA_DEV_OOB);
            } else {
                const int rb = a.fmt == CSA_KV_BF16 ? 2 * D : 656;
                erow = a.entries + re * (int64_t)rb;
            }
        }
    } else {
        wpos = (int64_t)w0 + (vk - n_sel);
        if (wpos < a.raw.first(b, a.seq_len[b])) {
            valid = false;
            if (lane == 0 && blockIdx.x == 0) flag(a.st, CSA_DEV_OOB);
        } else {
            wrow = a.kv + a.raw.row(b, wpos) * (int64_t)D;
        }
    }
    float2 v[NP];
#pragma unroll
    for (int u = 0; u < NP; u++) v[u] = make_float2(0.f, 0.f);
    if (erow) {
#pragma unroll
        for (int u = 0; u < NP; u++) {
            const int pi = lane + 32 * u;
            const int c = 2 * pi;
            if (a.fmt == CSA_KV_BF16) {
                v[u] = bf16x2_to_f32(*reinterpret_cast<const uint32_t*>(erow + 4 * pi));
            } else if (c < 512) {
                const float sc = *reinterpret_cast<const float*>(erow + 512 + 4 * (c >> 7));
                const uint32_t cc = *reinterpret_cast<const uint16_t*>(erow + c);
                v[u] = make_float2(e4m3_to_f32(cc & 0xFFu) * sc, e4m3_to_f32(cc >> 8) * sc);
            } else {
                v[u] = bf16x2_to_f32(*reinterpret_cast<const uint32_t*>(erow + 528 + 2 * (c - 512)));
            }
        }
    } else if (wrow) {
        float ss = 0.f;
#pragma unroll
        for (int u = 0; u < NP; u++) {
            v[u] = bf16x2_to_f32(*reinterpret_cast<const uint32_t*>(wrow + 2 * (lane + 32 * u)));
            ss += v[u].x * v[u].x + v[u].y * v[u].y;
        }
        ss = warp_sum(ss);
        const float r = rsqrtf(ss / (float)D + a.eps);
#pragma unroll
        for (int u = 0; u < NP; u++) {
            v[u].x *= r;
            v[u].y *= r;
            const int c = 2 * (lane + 32 * u);
            if (c >= D - kRopeDims) {
                float cs, sn;
                rope_cos_sin((double)wpos, (c - (D - kRopeDims)) >> 1, a.log2_theta, cs, sn);
                const float x = v[u].x, y = v[u].y;
                v[u].x = x * cs - y * sn;
                v[u].y = x * sn + y * cs;
            }
        }
    }
#pragma unroll
    for (int u = 0; u < NP; u++) {
        const int c = 2 * (lane + 32 * u);
        row[c] = v[u].x;
        row[c + 1] = v[u].y;
    }
    return valid;
}

template <int D>
__global__ void __launch_bounds__(256) attn_simt_kernel(AttnArgs a) {
    constexpr int LD = D + 1;
    constexpr int NR = D / 16;  // output channels per thread
    extern __shared__ float smem[];
    float* qs = smem;                       // [kHG][LD]
    float* ks = qs + kHG * LD;              // [kTK][LD]
    float* ss = ks + kTK * LD;              // [kHG][kTK]
    float* m_s = ss + kHG * kTK;            // [kHG]
    float* l_s = m_s + kHG;                 // [kHG]
    float* corr_s = l_s + kHG;              // [kHG]
    int* kval = reinterpret_cast<int*>(corr_s + kHG);  // [kTK]

    pdl_wait();
    pdl_trigger();
    const int qq = blockIdx.y;
    const int h0 = blockIdx.x * kHG;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = a.q_seq[qq];
    const int t = a.q_pos[qq];
    if (b < 0 || b >= a.B || t < 0 || (int64_t)t >= a.seq_len[b]) {
        if (tid == 0 && blockIdx.x == 0) flag(a.st, CSA_DEV_OOB);
        return;
    }
    const int n_vis = (t + 1) / a.m;
    const int n_sel = a.idx ? a.k : n_vis;
    const int w0 = t - a.W + 1 > 0 ? t - a.W + 1 : 0;
    const int n_win = a.W > 0 ? t - w0 + 1 : 0;
    const int n_keys = n_sel + n_win;

    // q heads: RoPE at t, one warp per head.
    for (int h = warp; h < kHG; h += 8) {
        const uint16_t* src = a.q + ((int64_t)qq * a.H + h0 + h) * D;
        for (int pi = lane; pi < D / 2; pi += 32) {
            float2 v = bf16x2_to_f32(*reinterpret_cast<const uint32_t*>(src + 2 * pi));
            const int c = 2 * pi;
            if (c >= D - kRopeDims) {
                float cs, sn;
                rope_cos_sin((double)t, (c - (D - kRopeDims)) >> 1, a.log2_theta, cs, sn);
                const float x = v.x, y = v.y;
                v.x = x * cs - y * sn;
                v.y = x * sn + y * cs;
            }
            qs[h * LD + c] = v.x;
            qs[h * LD + c + 1] = v.y;
        }
    }
    if (tid < kHG) {
        const float sk = a.sink[h0 + tid];
        m_s[tid] = sk;
        l_s[tid] = (sk == -INFINITY) ? 0.f : 1.f;
    }
    const int oh = tid >> 4, oc = tid & 15;  // output mapping: head oh, channels oc + 16r
    float o[NR];
#pragma unroll
    for (int r = 0; r < NR; r++) o[r] = 0.f;

    for (int base = 0; base < n_keys; base += kTK) {
        __syncthreads();  // previous tile fully consumed
        for (int j = warp; j < kTK; j += 8) {
            const int vk = base + j;
            bool valid = false;
            if (vk < n_keys) {
                valid = load_key<D>(a, b, t, n_vis, n_sel, w0, vk, ks + j * LD, lane);
            } else {
                for (int c = lane; c < D; c += 32) ks[j * LD + c] = 0.f;
            }
            if (lane == 0) kval[j] = valid ? 1 : 0;
        }
        __syncthreads();
        // logits: thread -> (head oh, keys oc and oc + 16)
#pragma unroll
        for (int half = 0; half < 2; half++) {
            const int j = oc + 16 * half;
            float d = 0.f;
            const float* qr = qs + oh * LD;
            const float* kr = ks + j * LD;
#pragma unroll 8
            for (int c = 0; c < D; c++) d = fmaf(qr[c], kr[c], d);
            ss[oh * kTK + j] = kval[j] ? d * a.scale : -INFINITY;
        }
        __syncthreads();
        if (tid < kHG) {
            const float m_old = m_s[tid];
            float tmax = -INFINITY;
            for (int j = 0; j < kTK; j++) tmax = fmaxf(tmax, ss[tid * kTK + j]);
            const float m_new = fmaxf(m_old, tmax);
            float corr = 1.f, lsum = 0.f;
            if (m_new != -INFINITY) {
                corr = expf(m_old - m_new);
                for (int j = 0; j < kTK; j++) {
                    const float p = expf(ss[tid * kTK + j] - m_new);
                    ss[tid * kTK + j] = p;
                    lsum += p;
                }
            } else {
                for (int j = 0; j < kTK; j++) ss[tid * kTK + j] = 0.f;
            }
            l_s[tid] = l_s[tid] * corr + lsum;
            m_s[tid] = m_new;
            corr_s[tid] = corr;
        }
        __syncthreads();
        const float cr = corr_s[oh];
#pragma unroll
        for (int r = 0; r < NR; r++) o[r] *= cr;
        for (int j = 0; j < kTK; j++) {
            const float p = ss[oh * kTK + j];
            const float* kr = ks + j * LD + oc;
#pragma unroll
            for (int r = 0; r < NR; r++) o[r] = fmaf(p, kr[16 * r], o[r]);
        }
    }
    __syncthreads();
    const float l = l_s[oh];
    const float inv = l > 0.f ? 1.f / l : 0.f;
    uint16_t* dst = a.out + ((int64_t)qq * a.H + h0 + oh) * D;
#pragma unroll
    for (int r = 0; r < NR; r++) {
        const int c = oc + 16 * r;
        float v = o[r] * inv;
        const float other = __shfl_xor_sync(0xffffffffu, v, 1);
        if (c >= D - kRopeDims) {
            float cs, sn;
            rope_cos_sin(-(double)t, (c - (D - kRopeDims)) >> 1, a.log2_theta, cs, sn);
            v = (c & 1) ? (other * sn + v * cs) : (v * cs - other * sn);
        }
        dst[c] = (uint16_t)f32_to_bf16_bits(v);
    }
}

template <int D>
static size_t attn_smem_bytes() {
    return sizeof(float) * ((size_t)(kHG + kTK) * (D + 1) + kHG * kTK + 3 * kHG) + sizeof(int) * kTK;
}

cudaError_t launch_attn_simt(const AttnArgs& a, int Q, int D, cudaStream_t stream) {
    if (Q == 0) return cudaSuccess;
    const dim3 grid(a.H / kHG, Q);
    LaunchScope scope(kKAttnSimt, stream);
    if (D == 128) {
        const size_t sm = attn_smem_bytes<128>();
        cudaFuncSetAttribute(attn_simt_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        return launch_pdl(attn_simt_kernel<128>, grid, dim3(256), sm, stream, a);
    } else {
        const size_t sm = attn_smem_bytes<576>();
        cudaFuncSetAttribute(attn_simt_kernel<576>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        return launch_pdl(attn_simt_kernel<576>, grid, dim3(256), sm, stream, a);
    }
    return cudaGetLastError();
}

}  // namespace csa
