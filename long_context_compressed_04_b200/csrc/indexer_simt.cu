// Step a3 (reference-grade CUDA-core path): lightning-indexer scores.
//
// "DeepSeek-V4 深度分析报告" 2.1 CSA: the lightning indexer scores every visible
// compressed entry for the query.  s_i = ks_i * sum_h (w_h*qs_h) * ReLU(q_h . k_i), with the
// heads accumulated by fmaf in ascending order in fp32.
//
// One thread per entry, the query's heads staged in shared memory as fp32.  This kernel
// serves shapes the tensor-core kernel does not take (d_I = 64, H_I not a multiple of 16);
// every e4m3 product is exact in fp32, so for integer-valued inputs both kernels give the
// same bits.
#include "launchers.cuh"

namespace csa {

template <int DI>
__global__ void __launch_bounds__(128) indexer_score_simt_kernel(
    const uint8_t* __restrict__ qI, const float* __restrict__ qs, const float* __restrict__ w,
    const uint8_t* __restrict__ kI, const float* __restrict__ ks, int64_t ent_rows,
    const int64_t* __restrict__ seq_len, const EntryRows er, const int32_t* __restrict__ q_seq,
    const int32_t* __restrict__ q_pos, int B, int HI, int m, int max_n,
    float* __restrict__ scores, int64_t ld, int32_t* __restrict__ dev_status) {
    extern __shared__ float smem[];
    pdl_wait();
    pdl_trigger();
    float* qf = smem;              // [HI][DI]
    float* wsh = smem + HI * DI;   // [HI]
    const int qq = blockIdx.y;
    const int b = q_seq[qq];
    const int t = q_pos[qq];
    if (b < 0 || b >= B || t < 0 || (int64_t)t >= seq_len[b]) {
        if (blockIdx.x == 0 && threadIdx.x == 0) flag(dev_status, CSA_DEV_OOB);
        return;
    }
    int n = (t + 1) / m;
    if (n > max_n) {
        if (blockIdx.x == 0 && threadIdx.x == 0) flag(dev_status, CSA_DEV_CAPACITY);
        n = max_n;
    }
    if (!er.bt) {
        const int64_t avail = ent_rows - er.ent_off[b];
        if ((int64_t)n > avail) {
            if (blockIdx.x == 0 && threadIdx.x == 0) flag(dev_status, CSA_DEV_OOB);
            n = avail > 0 ? (int)avail : 0;
        }
    }
    if ((int64_t)blockIdx.x * blockDim.x >= n) return;
    for (int x = threadIdx.x; x < HI * DI; x += blockDim.x)
        qf[x] = e4m3_to_f32(qI[(int64_t)qq * HI * DI + x]);
    for (int h = threadIdx.x; h < HI; h += blockDim.x)
        wsh[h] = w[(int64_t)qq * HI + h] * qs[(int64_t)qq * HI + h];
    __syncthreads();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int64_t row = er.row(b, i);
    if (row < 0 || row >= ent_rows) {   // a block outside the key store
        flag(dev_status, CSA_DEV_OOB);
        return;
    }
    float kf[DI];
    const uint4* src = reinterpret_cast<const uint4*>(kI + row * DI);
#pragma unroll
    for (int v = 0; v < DI / 16; v++) {
        const uint4 u = src[v];
        const uint32_t words[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int x = 0; x < 4; x++)
#pragma unroll
            for (int y = 0; y < 4; y++) kf[16 * v + 4 * x + y] = e4m3_to_f32((words[x] >> (8 * y)) & 0xFFu);
    }
    float acc = 0.f;
    for (int h = 0; h < HI; h++) {
        float d = 0.f;
#pragma unroll
        for (int c = 0; c < DI; c++) d = fmaf(qf[h * DI + c], kf[c], d);
        acc = fmaf(wsh[h], fmaxf(d, 0.f), acc);
    }
    const float s = acc * ks[row];
    if (s != s) flag(dev_status, CSA_DEV_NAN);
    scores[(int64_t)qq * ld + i] = s;
}

cudaError_t launch_indexer_simt(const uint8_t* qI, const float* qs, const float* w,
                                const uint8_t* kI, const float* ks, int64_t ent_rows,
                                const int64_t* seq_len,
                                const EntryRows& er, const int32_t* q_seq, const int32_t* q_pos, int Q, int B,
                                int HI, int dI, int m, int max_n, float* scores, int64_t ld,
                                int32_t* st, cudaStream_t stream) {
    if (Q == 0 || max_n == 0) return cudaSuccess;
    const dim3 grid((max_n + 127) / 128, Q);
    const size_t smem = sizeof(float) * (size_t)(HI * dI + HI);
    LaunchScope scope(kKIndexerSimt, stream);
    if (dI == 64) {
        return launch_pdl(indexer_score_simt_kernel<64>, grid, dim3(128), smem, stream, qI, qs, w,
                          kI, ks, ent_rows, seq_len, er, q_seq, q_pos, B, HI, m, max_n,
                          scores, ld, st);
    } else {
        cudaFuncSetAttribute(indexer_score_simt_kernel<128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        return launch_pdl(indexer_score_simt_kernel<128>, grid, dim3(128), smem, stream, qI, qs,
                          w, kI, ks, ent_rows, seq_len, er, q_seq, q_pos, B, HI, m, max_n,
                          scores, ld, st);
    }
    return cudaGetLastError();
}

}  // namespace csa
