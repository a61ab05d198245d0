// simt.cuh -- plain CUDA-core kernels for every product of the packed LoRA
// forward/backward.  This is the fp32 path (true fp32 FMA, no TF32) and the
// bf16 cross-check path; the bf16 production path is the tensor-core one.
#pragma once
#include <cuda_bf16.h>
#include "plan.cuh"

namespace plora {

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// One 64x64 output tile per block, 256 threads, 4x4 outputs per thread, K in steps of 16.
// The block's op is found by binary search over the ops' first block indices.
template <typename T>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const SimtOp* __restrict__ ops, int n_ops) {
    __shared__ float As[16][65];
    __shared__ float Bs[16][65];
    int lo = 0, hi = n_ops - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (ops[mid].tile_begin <= (int)blockIdx.x) lo = mid; else hi = mid - 1;
    }
    const SimtOp op = ops[lo];
    const int t = blockIdx.x - op.tile_begin;
    const int m0 = (t / op.tiles_n) * 64, n0 = (t % op.tiles_n) * 64;
    const T* A = static_cast<const T*>(op.A);
    const T* B = static_cast<const T*>(op.B);
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < op.K; k0 += 16) {
        for (int e = threadIdx.x; e < 1024; e += 256) {
            int mm, kk;
            if (op.a_sk == 1) { mm = e >> 4; kk = e & 15; } else { kk = e >> 6; mm = e & 63; }
            const int m = m0 + mm, k = k0 + kk;
            As[kk][mm] = (m < op.M && k < op.K) ? to_f<T>(A[(int64_t)m * op.a_sm + (int64_t)k * op.a_sk]) : 0.f;
            int nn, kb;
            if (op.b_sk == 1) { nn = e >> 4; kb = e & 15; } else { kb = e >> 6; nn = e & 63; }
            const int n = n0 + nn, k2 = k0 + kb;
            Bs[kb][nn] = (n < op.N && k2 < op.K) ? to_f<T>(B[(int64_t)k2 * op.b_sk + (int64_t)n * op.b_sn]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty + 16 * i;
        if (m >= op.M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx + 16 * j;
            if (n >= op.N) continue;
            const int64_t ci = (int64_t)m * op.c_sm + (int64_t)n * op.c_sn;
            float v = op.alpha * acc[i][j];
            if (op.c_fp32) {
                float* C = static_cast<float*>(op.C);
                if (op.accumulate) v += C[ci];
                C[ci] = v;
            } else {
                T* C = static_cast<T*>(op.C);
                if (op.accumulate) v += to_f<T>(C[ci]);
                C[ci] = from_f<T>(v);
            }
        }
    }
}

// Copy adapter i's saved H block ([n][rp] rows of the saved buffer, pitch RP) to fp32 [n][rank].
template <typename T>
// out[t][p rank + k] = saved row h_row + t, column p rblk + k (block p of nblk output blocks).
__global__ void unpack_saved_kernel(const T* __restrict__ saved, int64_t h_row, int RP, int n, int rank,
                                    int nblk, int rblk, float* __restrict__ out) {
    const int width = nblk * rank;
    const int64_t total = (int64_t)n * width;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = e / width;
        const int j = (int)(e - t * width);
        const int pb = j / rank;
        const int k = j - pb * rank;
        out[e] = to_f<T>(saved[(h_row + t) * RP + pb * rblk + k]);
    }
}

}  // namespace plora
