// Bandwidth-bound helper kernels: deterministic column sums (the bias
// gradients), the activation rebuild for recompute, and small utilities.
#pragma once

#include "gemm_tc.cuh"

namespace tpmlp {

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// Column sums, pass 1, one block's share. Block (32, 8): lane x covers
// columns [bx·256 + 8x, +8), row phase y walks rows chunk_begin + y, +8, ...
// of chunk `chunk`; the 8 phases are then added in order y = 0..7 and the
// chunk's sums written to partial[chunk][:]. Fixed assignment and fixed
// order: the result is bit-reproducible.
template <typename T, bool VEC>
__device__ __forceinline__ void colsum_partial_block(const T* __restrict__ X, int64_t R, int64_t C,
                                                     int64_t rows_per_chunk,
                                                     float* __restrict__ partial, int bx, int chunk) {
    __shared__ float red[8][256];
    const int64_t c0 = static_cast<int64_t>(bx) * 256 + threadIdx.x * 8;
    const int64_t r_begin = static_cast<int64_t>(chunk) * rows_per_chunk;
    const int64_t r_end = min(R, r_begin + rows_per_chunk);
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (VEC && c0 < C) {
        // C % 8 == 0 and X 16-byte aligned: 8 columns are 16 (bf16) or 32 (fp32)
        // bytes. Rows are visited in the same order as the scalar loop, but
        // the loads of up to kU rows (128 bytes per thread) are issued before
        // their additions so that many are in flight at once.
        constexpr int kU = sizeof(T) == 2 ? 8 : 4;
        int64_t r = r_begin + threadIdx.y;
        for (; r + 8 * (kU - 1) < r_end; r += 8 * kU) {
            if constexpr (sizeof(T) == 2) {
                uint4 raw[kU];
#pragma unroll
                for (int u = 0; u < kU; ++u)
                    raw[u] = __ldg(reinterpret_cast<const uint4*>(X + (r + 8 * u) * C + c0));
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    float f[8];
                    unpack_bf16x8(raw[u], f);
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[i] += f[i];
                }
            } else {
                float4 lo[kU], hi[kU];
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    lo[u] = __ldg(reinterpret_cast<const float4*>(X + (r + 8 * u) * C + c0));
                    hi[u] = __ldg(reinterpret_cast<const float4*>(X + (r + 8 * u) * C + c0) + 1);
                }
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    acc[0] += lo[u].x; acc[1] += lo[u].y; acc[2] += lo[u].z; acc[3] += lo[u].w;
                    acc[4] += hi[u].x; acc[5] += hi[u].y; acc[6] += hi[u].z; acc[7] += hi[u].w;
                }
            }
        }
        for (; r < r_end; r += 8) {
            const T* row = X + r * C + c0;
            if constexpr (sizeof(T) == 2) {
                float f[8];
                unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(row)), f);
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] += f[i];
            } else {
                const float4 lo = __ldg(reinterpret_cast<const float4*>(row));
                const float4 hi = __ldg(reinterpret_cast<const float4*>(row) + 1);
                acc[0] += lo.x; acc[1] += lo.y; acc[2] += lo.z; acc[3] += lo.w;
                acc[4] += hi.x; acc[5] += hi.y; acc[6] += hi.z; acc[7] += hi.w;
            }
        }
    } else if (!VEC) {
        for (int64_t r = r_begin + threadIdx.y; r < r_end; r += 8) {
            const T* row = X + r * C;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (c0 + i < C) acc[i] += to_f32<T>(row[c0 + i]);
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) red[threadIdx.y][threadIdx.x * 8 + i] = acc[i];
    __syncthreads();
    const int t = threadIdx.y * 32 + threadIdx.x;  // 0..255: one column each
    const int64_t c = static_cast<int64_t>(bx) * 256 + t;
    if (c < C) {
        float s = red[0][t];
        for (int y = 1; y < 8; ++y) s += red[y][t];
        partial[static_cast<int64_t>(chunk) * C + c] = s;
    }
}

// Pass 1 of one R × C matrix: grid (⌈C/256⌉, chunks).
template <typename T, bool VEC>
__global__ void __launch_bounds__(256) colsum_partial_kernel(const T* __restrict__ X, int64_t R,
                                                            int64_t C, int64_t rows_per_chunk,
                                                            float* __restrict__ partial) {
    grid_dep_wait();  // every input may come from the predecessor kernel
    grid_dep_launch();
    colsum_partial_block<T, VEC>(X, R, C, rows_per_chunk, partial, static_cast<int>(blockIdx.x),
                                 static_cast<int>(blockIdx.y));
}

// Pass 1 of two matrices with the same R (column blocks of X1 first, then
// of X2: grid (⌈C1/256⌉ + ⌈C2/256⌉, chunks)); each column's sum is the one
// colsum_partial_kernel computes.
template <typename T, bool VEC>
__global__ void __launch_bounds__(256) colsum_partial2_kernel(const T* __restrict__ X1, int64_t C1,
                                                             float* __restrict__ partial1,
                                                             const T* __restrict__ X2, int64_t C2,
                                                             float* __restrict__ partial2, int64_t R,
                                                             int64_t rows_per_chunk) {
    grid_dep_wait();
    grid_dep_launch();
    const int nb1 = static_cast<int>((C1 + 255) / 256);
    const int bx = static_cast<int>(blockIdx.x), by = static_cast<int>(blockIdx.y);
    if (bx < nb1)
        colsum_partial_block<T, VEC>(X1, R, C1, rows_per_chunk, partial1, bx, by);
    else
        colsum_partial_block<T, VEC>(X2, R, C2, rows_per_chunk, partial2, bx - nb1, by);
}

// Column sums, pass 2: out[c] = Σ over chunks of partial[chunk][c]. Block
// (32, 8): x picks one of 32 consecutive columns (coalesced reads), y one of 8
// contiguous chunk groups; each thread adds its group's chunks in ascending
// order, then the 8 group sums are added in ascending group order. Fixed
// assignment and order: bit-reproducible.
__device__ __forceinline__ void colsum_final_block(const float* __restrict__ partial, int chunks,
                                                   int64_t C, float* __restrict__ out, int64_t bx) {
    __shared__ float grp[8][32];
    const int64_t c = bx * 32 + threadIdx.x;
    const int per = (chunks + 7) / 8;
    const int k0 = threadIdx.y * per;
    const int k1 = min(chunks, k0 + per);
    float s = 0.0f;
    if (c < C) {
        int k = k0;
        for (; k + 8 <= k1; k += 8) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = partial[(k + u) * C + c];
#pragma unroll
            for (int u = 0; u < 8; ++u) s += v[u];
        }
        for (; k < k1; ++k) s += partial[k * C + c];
    }
    grp[threadIdx.y][threadIdx.x] = s;
    __syncthreads();
    if (threadIdx.y == 0 && c < C) {
        float t = grp[0][threadIdx.x];
#pragma unroll
        for (int y = 1; y < 8; ++y) t += grp[y][threadIdx.x];
        out[c] = t;
    }
}

// Pass 2 of one matrix: grid ⌈C/32⌉.
__global__ void __launch_bounds__(256) colsum_final_kernel(const float* __restrict__ partial,
                                                          int chunks, int64_t C,
                                                          float* __restrict__ out) {
    grid_dep_wait();  // every input may come from the predecessor kernel
    grid_dep_launch();
    colsum_final_block(partial, chunks, C, out, blockIdx.x);
}

// Pass 2 of two matrices (the column blocks of the first, then of the
// second: grid ⌈C1/32⌉ + ⌈C2/32⌉); each sum is the one colsum_final_kernel
// computes.
__global__ void __launch_bounds__(256) colsum_final2_kernel(const float* __restrict__ partial1,
                                                           int chunks1, int64_t C1,
                                                           float* __restrict__ out1,
                                                           const float* __restrict__ partial2,
                                                           int chunks2, int64_t C2,
                                                           float* __restrict__ out2) {
    grid_dep_wait();
    grid_dep_launch();
    const int64_t nb1 = (C1 + 31) / 32;
    if (blockIdx.x < nb1)
        colsum_final_block(partial1, chunks1, C1, out1, blockIdx.x);
    else
        colsum_final_block(partial2, chunks2, C2, out2, blockIdx.x - nb1);
}

// GeLU and GeLU′ of n values with each form the library uses:
// 0 = exact GeLU as in the tensor-core epilogues (Hastings erf), 1 = exact
// GeLU through CUDA's erff/expf, 2 = tanh form as in the tensor-core
// epilogues (½(1 + tanh u) as a logistic function of 2u), 3 = tanh form
// through CUDA's tanhf. Forms 0 and 2 run in packed pairs like the epilogues.
__global__ void eval_activation_kernel(const float* __restrict__ x, float* __restrict__ y,
                                       float* __restrict__ dy, int64_t n, int form) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float v = x[i];
        if (form == 0 || form == 2) {
            // the packed pair (x[2k], x[2k+1]) as the epilogues form it, so
            // both halves of the packed arithmetic are checked
            const int64_t j = i ^ 1;
            const float w = j < n ? x[j] : v;
            const bool hi = (i & 1) != 0;
            const float a = hi ? w : v, b = hi ? v : w;
            float p0, p1, q0, q1;
            if (form == 0) {
                gelu_fast_x2(a, b, p0, p1);
                gelu_grad_fast_x2(a, b, q0, q1);
            } else {
                gelu_tanh_fast_x2(a, b, p0, p1);
                gelu_tanh_grad_fast_x2(a, b, q0, q1);
            }
            y[i] = hi ? p1 : p0;
            dy[i] = hi ? q1 : q0;
        } else if (form == 1) {
            y[i] = gelu_f32(v);
            dy[i] = gelu_grad_f32(v);
        } else {
            y[i] = gelu_tanh_f32(v);
            dy[i] = gelu_tanh_grad_f32(v);
        }
    }
}

// Activation recompute: Y[i] = act(H[i]) for i < n. bf16 uses the
// tensor-core epilogues' forms, fp32 the plain path's (CUDA erff / tanhf).
template <bool TANH>
__device__ __forceinline__ uint4 act_bf16x8(uint4 raw) {
    float f[8];
    unpack_bf16x8(raw, f);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        if constexpr (TANH) gelu_tanh_fast_x2(f[i], f[i + 1], f[i], f[i + 1]);
        else gelu_fast_x2(f[i], f[i + 1], f[i], f[i + 1]);
    }
    uint4 o;
    o.x = pack_bf16x2(f[0], f[1]);
    o.y = pack_bf16x2(f[2], f[3]);
    o.z = pack_bf16x2(f[4], f[5]);
    o.w = pack_bf16x2(f[6], f[7]);
    return o;
}

template <bool TANH>
__device__ __forceinline__ float4 act_f32x4(float4 v) {
    v.x = TANH ? gelu_tanh_f32(v.x) : gelu_f32(v.x);
    v.y = TANH ? gelu_tanh_f32(v.y) : gelu_f32(v.y);
    v.z = TANH ? gelu_tanh_f32(v.z) : gelu_f32(v.z);
    v.w = TANH ? gelu_tanh_f32(v.w) : gelu_f32(v.w);
    return v;
}

// VEC: n % 8 == 0 and both pointers 16-byte aligned. 8 elements form one
// group (16 bytes of bf16, 32 of fp32); a thread-iteration takes two groups a
// grid stride apart and issues both loads before computing either, so that
// more bytes are in flight per SM.
template <typename T, bool TANH, bool VEC>
__global__ void __launch_bounds__(256, 8) recompute_act_kernel(const T* __restrict__ H,
                                                           T* __restrict__ Y, int64_t n) {
    grid_dep_wait();  // every input may come from the predecessor kernel
    grid_dep_launch();
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t first = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    if constexpr (VEC) {
        const int64_t groups = n / 8;
        for (int64_t g = first; g < groups; g += 2 * stride) {
            const int64_t g2 = g + stride;
            const bool second = g2 < groups;
            if constexpr (sizeof(T) == 2) {
                const uint4* h = reinterpret_cast<const uint4*>(H);
                uint4* y = reinterpret_cast<uint4*>(Y);
                const uint4 r0 = __ldg(h + g);
                uint4 r1 = make_uint4(0, 0, 0, 0);
                if (second) r1 = __ldg(h + g2);
                y[g] = act_bf16x8<TANH>(r0);
                if (second) y[g2] = act_bf16x8<TANH>(r1);
            } else {
                const float4* h = reinterpret_cast<const float4*>(H);
                float4* y = reinterpret_cast<float4*>(Y);
                const float4 a0 = __ldg(h + 2 * g), a1 = __ldg(h + 2 * g + 1);
                float4 b0 = make_float4(0, 0, 0, 0), b1 = b0;
                if (second) {
                    b0 = __ldg(h + 2 * g2);
                    b1 = __ldg(h + 2 * g2 + 1);
                }
                y[2 * g] = act_f32x4<TANH>(a0);
                y[2 * g + 1] = act_f32x4<TANH>(a1);
                if (second) {
                    y[2 * g2] = act_f32x4<TANH>(b0);
                    y[2 * g2 + 1] = act_f32x4<TANH>(b1);
                }
            }
        }
    } else {
        for (int64_t i = first; i < n; i += stride) {
            const float x = to_f32<T>(H[i]);
            float y;
            if constexpr (sizeof(T) == 2) {
                float unused;
                if constexpr (TANH) gelu_tanh_fast_x2(x, x, y, unused);
                else gelu_fast_x2(x, x, y, unused);
            } else {
                y = TANH ? gelu_tanh_f32(x) : gelu_f32(x);
            }
            if constexpr (sizeof(T) == 2) Y[i] = __float2bfloat16_rn(y);
            else Y[i] = y;
        }
    }
}

__global__ void zero_f32_kernel(float* __restrict__ p, int64_t n) {
    grid_dep_wait();  // every input may come from the predecessor kernel
    grid_dep_launch();
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        p[i] = 0.0f;
}

// A kernel that waits, bounded, on an mbarrier that nothing completes:
// exercises the timeout path (status word set, clean return).
__global__ void wait_selftest_kernel(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (!mbar_wait_bounded(smem_u32(&bar), 0, &abort_flag, limit_ns)) raise_timeout(&abort_flag);
    }
    __syncthreads();
}

}  // namespace tpmlp
