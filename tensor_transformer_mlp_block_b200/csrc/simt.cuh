// Plain CUDA-core GEMM with the same fused epilogues as the tensor-core path.
//
// Serves the fp32 dtype (true fp32 FFMA, no TF32: each output is one fp32
// accumulator updated with fmaf over k in ascending order) and bf16 shapes
// the tensor-memory accelerator cannot describe (h or F not a multiple of 8).
// Operands are addressed through explicit strides, so one kernel covers
// every transposition the block needs.
#pragma once

#include "gemm_tc.cuh"

namespace tpmlp {

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

template <typename T>
__device__ __forceinline__ float ld_f32(const T* p);
template <>
__device__ __forceinline__ float ld_f32<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ld_f32<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

struct SimtArgs {
    int M, N, K;
    const void* A;  // Aop(m, k) = A[m·sam + k·sak]
    int64_t sam, sak;
    const void* B;  // Bop(k, n) = B[k·sbk + n·sbn]
    int64_t sbk, sbn;
    void* out0;
    void* out1;
    int64_t ld_out;
    const void* bias;  // length N, element type T, may be null
    const void* aux;   // saved H for EPI_DGELU
};

// 16 × 16 outputs per block, one per thread; 16-wide k tiles staged in
// shared memory. Each output's sum runs over k = 0..K-1 in order.
template <typename T, int EPI>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const SimtArgs g) {
    __shared__ float sA[16][17];
    __shared__ float sB[16][17];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int m = blockIdx.y * 16 + ty;
    const int n = blockIdx.x * 16 + tx;
    const T* A = static_cast<const T*>(g.A);
    const T* B = static_cast<const T*>(g.B);
    float acc = 0.0f;
    for (int k0 = 0; k0 < g.K; k0 += 16) {
        {
            const int mm = blockIdx.y * 16 + ty, kk = k0 + tx;
            sA[ty][tx] = (mm < g.M && kk < g.K) ? ld_f32<T>(A + mm * g.sam + kk * g.sak) : 0.0f;
            const int kb = k0 + ty, nn = blockIdx.x * 16 + tx;
            sB[ty][tx] = (kb < g.K && nn < g.N) ? ld_f32<T>(B + kb * g.sbk + nn * g.sbn) : 0.0f;
        }
        __syncthreads();
        const int kn = min(16, g.K - k0);
        for (int k = 0; k < kn; ++k) acc = fmaf(sA[ty][k], sB[k][tx], acc);
        __syncthreads();
    }
    if (m >= g.M || n >= g.N) return;
    const int64_t off = static_cast<int64_t>(m) * g.ld_out + n;
    if constexpr (EPI == EPI_F32) {
        static_cast<float*>(g.out0)[off] = acc;
    } else {
        float v = acc;
        if constexpr (EpiTraits<EPI>::kBias) {
            if (g.bias != nullptr) v += ld_f32<T>(static_cast<const T*>(g.bias) + n);
        }
        if constexpr (EpiTraits<EPI>::kDAct) {
            const float hv = ld_f32<T>(static_cast<const T*>(g.aux) + off);
            v *= EpiTraits<EPI>::kTanh ? gelu_tanh_grad_f32(hv) : gelu_grad_f32(hv);
        }
        static_cast<T*>(g.out0)[off] = from_f32<T>(v);
        if constexpr (EpiTraits<EPI>::kAct)
            static_cast<T*>(g.out1)[off] = from_f32<T>(EpiTraits<EPI>::kTanh ? gelu_tanh_f32(v) : gelu_f32(v));
    }
}

}  // namespace tpmlp
