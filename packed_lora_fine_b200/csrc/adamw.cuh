// adamw.cuh -- one AdamW step for every adapter of a packed job in a single launch.
//
// Every adapter's A and B (with their fp32 master copies, moments and fp32 gradients) are
// flattened into segments; the launch is a grid of blocks over fixed-size chunks of all
// segments, so adapters of any rank share the launch and the GPU stays full.  The update is
// elementwise and HBM-bound: per element it reads g, m, v, p (16 B) and writes m, v, p and
// the parameter copy (12 B + 2 B for bf16).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace plora {

constexpr int kAdamwChunk = 8192;   // elements per block

// One contiguous tensor of one adapter (its A or its B).
struct AdamwSeg {
    float* p;            // fp32 master parameters
    float* m;
    float* v;
    const float* g;      // fp32 gradient
    void* out;           // the layer's parameter copy (bf16), or nullptr when p is the parameter
    int64_t n;           // elements (a multiple of 4)
    float decay;         // 1 - lr * weight_decay
    float step_size;     // lr / (1 - beta1^t)
    float beta1, beta2;
    float inv_sqrt_bc2;  // 1 / sqrt(1 - beta2^t)
    float eps;
};
static_assert(sizeof(AdamwSeg) % 8 == 0, "AdamwSeg layout");

struct AdamwChunk {
    int32_t seg;
    int32_t pad_;
    int64_t start;       // first element of the chunk in the segment
};
static_assert(sizeof(AdamwChunk) == 16, "AdamwChunk layout");

__device__ __forceinline__ float adamw_elem(float p, float& m, float& v, float g, const AdamwSeg& s) {
    p = p * s.decay;
    m = s.beta1 * m + (1.f - s.beta1) * g;
    v = s.beta2 * v + (1.f - s.beta2) * g * g;
    const float denom = sqrtf(v) * s.inv_sqrt_bc2 + s.eps;
    return p - s.step_size * (m / denom);
}

__global__ void __launch_bounds__(256) adamw_kernel(const AdamwSeg* __restrict__ segs,
                                                    const AdamwChunk* __restrict__ chunks) {
    const AdamwChunk c = chunks[blockIdx.x];
    const AdamwSeg s = segs[c.seg];
    const int64_t end = s.n < c.start + kAdamwChunk ? s.n : c.start + kAdamwChunk;
    for (int64_t e = c.start + 4 * (int64_t)threadIdx.x; e < end; e += 4 * (int64_t)blockDim.x) {
        float4 p = *reinterpret_cast<const float4*>(s.p + e);
        float4 m = *reinterpret_cast<const float4*>(s.m + e);
        float4 v = *reinterpret_cast<const float4*>(s.v + e);
        const float4 g = *reinterpret_cast<const float4*>(s.g + e);
        p.x = adamw_elem(p.x, m.x, v.x, g.x, s);
        p.y = adamw_elem(p.y, m.y, v.y, g.y, s);
        p.z = adamw_elem(p.z, m.z, v.z, g.z, s);
        p.w = adamw_elem(p.w, m.w, v.w, g.w, s);
        *reinterpret_cast<float4*>(s.p + e) = p;
        *reinterpret_cast<float4*>(s.m + e) = m;
        *reinterpret_cast<float4*>(s.v + e) = v;
        if (s.out) {
            __nv_bfloat162 lo = __floats2bfloat162_rn(p.x, p.y);
            __nv_bfloat162 hi = __floats2bfloat162_rn(p.z, p.w);
            uint2 w;
            w.x = *reinterpret_cast<uint32_t*>(&lo);
            w.y = *reinterpret_cast<uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(s.out) + e) = w;
        }
    }
}

}  // namespace plora
