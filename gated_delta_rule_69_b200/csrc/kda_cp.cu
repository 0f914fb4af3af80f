// Context parallelism across devices: the combine step.
//
// One sequence cut into segments, one per device.  A segment's effect on the
// state it receives is the product of its tokens' transitions
// M_t = (I - beta_t k_t k_t^T) Diag(alpha_t), applied to the incoming state,
// plus the state it generates from zero, S~ (course page "Attention lineaire
// et recurrence", section "Verification de comprehension": each segment
// carries its cumulative transition M and its locally generated state S~).
// A device that holds segment r therefore starts from
//     S_in(0) = S_0,   S_in(i + 1) = M_i S_in(i) + S~_i   (i < r)
// which this kernel forms from the gathered (M_i, S~_i) of the segments
// before it.  fp32 on CUDA cores: d_k x d_k x d_v per step, a few steps.
//
// Grid: heads x (d_v / 32) column blocks (a product acts on columns
// independently).  A CTA keeps M_i (d_k x d_k) and its 32 columns of S in
// shared memory; thread t computes rows t / 2 (two threads per row, 16
// columns each).
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kCpThreads = 256;
constexpr int kCpCols = 32;

__global__ void __launch_bounds__(kCpThreads)
kda_cp_combine_kernel(const float *__restrict__ M, const float *__restrict__ St,
                      const float *__restrict__ S0, float *__restrict__ S_out, int n_prev,
                      int H, int dk, int dv) {
    extern __shared__ float sh[];
    float *sM = sh;                      // dk x dk
    float *sS = sM + dk * dk;            // dk x kCpCols
    const int h = blockIdx.x;
    const int j0 = blockIdx.y * kCpCols;
    const int tid = threadIdx.x;
    const size_t soff = (size_t)h * dk * dv;
    for (int idx = tid; idx < dk * kCpCols; idx += kCpThreads) {
        const int c = idx / kCpCols, j = idx % kCpCols;
        sS[idx] = S0 ? S0[soff + (size_t)c * dv + j0 + j] : 0.f;
    }
    const int row = tid >> 1, cb = (tid & 1) * 16;
    for (int i = 0; i < n_prev; ++i) {
        const float *Mi = M + ((size_t)i * H + h) * dk * dk;
        const float *Si = St + ((size_t)i * H + h) * dk * dv;
        __syncthreads();   // sS final for this step; sM free
        for (int idx = tid; idx < dk * dk; idx += kCpThreads) sM[idx] = Mi[idx];
        __syncthreads();
        float acc[16];
        const bool active = row < dk;
        if (active) {
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[e] = Si[(size_t)row * dv + j0 + cb + e];
            for (int c = 0; c < dk; ++c) {
                const float m = sM[row * dk + c];
                const float *s = sS + c * kCpCols + cb;
#pragma unroll
                for (int e = 0; e < 16; ++e) acc[e] = fmaf(m, s[e], acc[e]);
            }
        }
        __syncthreads();   // every read of sS done before it is overwritten
        if (active) {
#pragma unroll
            for (int e = 0; e < 16; ++e) sS[row * kCpCols + cb + e] = acc[e];
        }
    }
    __syncthreads();
    for (int idx = tid; idx < dk * kCpCols; idx += kCpThreads) {
        const int c = idx / kCpCols, j = idx % kCpCols;
        S_out[soff + (size_t)c * dv + j0 + j] = sS[idx];
    }
}

}  // namespace

cudaError_t launch_cp_combine(const float *M, const float *S_tilde, const float *S0, float *S_out,
                              int n_prev, int H, int dk, int dv, cudaStream_t stream) {
    const size_t smem = (size_t)(dk * dk + dk * kCpCols) * sizeof(float);
    const cudaError_t e = set_max_dynamic_smem((const void *)kda_cp_combine_kernel,
                                               (int)((128 * 128 + 128 * kCpCols) * sizeof(float)));
    if (e != cudaSuccess) return e;
    kda_cp_combine_kernel<<<dim3(H, dv / kCpCols), kCpThreads, smem, stream>>>(M, S_tilde, S0, S_out,
                                                                            n_prev, H, dk, dv);
    return cudaGetLastError();
}

}  // namespace kda
