// The elementwise stages around the projection GEMMs of the mixer with its
// producers (conv output -> x_proj -> [dt_low | B | C] -> dt_proj -> scan):
//
//   conv_silu_kernel   u_t = SiLU(conv_b + sum_k conv_w[k] x_{t-3+k}), bf16, the
//                      A operand of x_proj (the scan recomputes u itself);
//   xproj_epilogue_kernel  sums x_proj's split-K partials and splits each row
//                      into dt_low (dt_rank wide), B_t and C_t (d_state each),
//                      each optionally RMS-normalised over its own width (the
//                      Jamba report puts RMSNorm inside the Mamba layer, on
//                      its internal activations), stored in bf16.
// Both are HBM-streaming kernels: every access of a warp is one contiguous span.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "mixer_common.cuh"

namespace mm {

constexpr int kConvTokens = 32;   // tokens one thread walks with its window in registers
#ifndef MM_CONV_STEP
#define MM_CONV_STEP 4             // tokens whose x rows one thread requests at once (8 and 16 measured slower)
#endif

// One thread: 8 consecutive channels of one sequence over kConvTokens tokens.
__global__ void __launch_bounds__(128)
conv_silu_kernel(const __nv_bfloat16* __restrict__ xz, const float* __restrict__ conv_w,
                 const float* __restrict__ conv_b, const __nv_bfloat16* __restrict__ cs_in,
                 __nv_bfloat16* __restrict__ u, int64_t L, int D)
{
    const int oct = blockIdx.x * blockDim.x + threadIdx.x;      // channel octet
    if (oct * 8 >= D) return;
    const int b = blockIdx.z;
    const int64_t t0 = static_cast<int64_t>(blockIdx.y) * kConvTokens;
    const int d0 = oct * 8;
    float w[8][4], cb[8], win[8][3];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const float4 wv = *reinterpret_cast<const float4*>(conv_w + static_cast<int64_t>(d0 + c) * 4);
        w[c][0] = wv.x; w[c][1] = wv.y; w[c][2] = wv.z; w[c][3] = wv.w;
        cb[c] = conv_b ? conv_b[d0 + c] : 0.0f;
    }
    const __nv_bfloat16* xrow = xz + static_cast<int64_t>(b) * L * 2 * D + d0;
    // the three raw x before t0: earlier tokens, or the carried window (oldest first)
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int64_t t = t0 - 3 + j;
        if (t >= 0) {
            const uint4 v = *reinterpret_cast<const uint4*>(xrow + t * 2 * D);
            const uint32_t wds[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int c = 0; c < 8; ++c)
                win[c][j] = __uint_as_float((c & 1) ? (wds[c >> 1] & 0xffff0000u) : (wds[c >> 1] << 16));
        } else {
#pragma unroll
            for (int c = 0; c < 8; ++c)
                win[c][j] = cs_in ? Act<__nv_bfloat16>::to_f32(cs_in[(static_cast<int64_t>(b) * D + d0 + c) * 3 + (t + 3)])
                                  : 0.0f;
        }
    }
    const int64_t t_end = min(L, t0 + kConvTokens);
    __nv_bfloat16* urow = u + static_cast<int64_t>(b) * L * D + d0;
    // kStep tokens per step: their rows of x are requested together, so that
    // many loads are in flight per thread instead of one
    constexpr int kStep = MM_CONV_STEP;
    for (int64_t tb = t0; tb < t_end; tb += kStep) {
        uint4 xv[kStep];
#pragma unroll
        for (int j = 0; j < kStep; ++j)
            xv[j] = tb + j < t_end ? *reinterpret_cast<const uint4*>(xrow + (tb + j) * 2 * D) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int j = 0; j < kStep; ++j) {
            if (tb + j >= t_end) break;
            const uint32_t wds[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
            float o[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float x = __uint_as_float((c & 1) ? (wds[c >> 1] & 0xffff0000u) : (wds[c >> 1] << 16));
                float pre = cb[c];
                pre = fmaf(w[c][0], win[c][0], pre);
                pre = fmaf(w[c][1], win[c][1], pre);
                pre = fmaf(w[c][2], win[c][2], pre);
                pre = fmaf(w[c][3], x, pre);
                o[c] = MathFast::silu(pre);
                win[c][0] = win[c][1];
                win[c][1] = win[c][2];
                win[c][2] = x;
            }
            uint4 r;
            r.x = pack_bf16x2(o[0], o[1]);
            r.y = pack_bf16x2(o[2], o[3]);
            r.z = pack_bf16x2(o[4], o[5]);
            r.w = pack_bf16x2(o[6], o[7]);
            *reinterpret_cast<uint4*>(urow + (tb + j) * D) = r;
        }
    }
}

// One warp per row of x_proj's output (dt_rank + 2 d_state = R + 32 columns,
// R a multiple of 32): lane l holds columns l + 32 j.  Columns 0..R-1 are
// dt_low, R..R+15 are B, R+16..R+31 are C.
__global__ void __launch_bounds__(256)
xproj_epilogue_kernel(const float* __restrict__ part, int splits, int64_t split_stride, int64_t M, int R,
                      const float* __restrict__ dt_norm_w, const float* __restrict__ b_norm_w,
                      const float* __restrict__ c_norm_w, float eps,
                      __nv_bfloat16* __restrict__ dt_low, __nv_bfloat16* __restrict__ Bo, __nv_bfloat16* __restrict__ Co)
{
    const int lane = threadIdx.x & 31;
    const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (row >= M) return;
    const int NC = R + 32;
    const int J = R / 32;
    // the first 8 x 32 columns of dt_low stay in registers for the normalised store
    float v[8];
    float ss_dt = 0.0f;
    auto col_sum = [&](int j) {
        float acc = 0.0f;
        for (int s = 0; s < splits; ++s) acc += part[s * split_stride + row * NC + lane + 32 * j];
        return acc;
    };
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        v[j] = 0.0f;
        if (j < J) {
            const float acc = col_sum(j);
            ss_dt = fmaf(acc, acc, ss_dt);
            v[j] = acc;
            // dt_low: stored now unless it is to be normalised (then after the row's sum)
            if (!dt_norm_w) dt_low[row * R + lane + 32 * j] = __float2bfloat16_rn(acc);
        }
    }
    for (int j = 8; j < J; ++j) {
        const float acc = col_sum(j);
        ss_dt = fmaf(acc, acc, ss_dt);
        if (!dt_norm_w) dt_low[row * R + lane + 32 * j] = __float2bfloat16_rn(acc);
    }
    const float vbc = col_sum(J);
    // B (lanes 0..15) and C (lanes 16..31): sums of squares within each half-warp
    float ss_bc = vbc * vbc;
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) ss_bc += __shfl_xor_sync(kFull, ss_bc, o);
    const bool is_c = lane >= 16;
    const float* wbc = is_c ? c_norm_w : b_norm_w;
    float bc = vbc;
    if (wbc) bc *= rsqrtf(fmaf(ss_bc, 1.0f / 16.0f, eps)) * wbc[lane & 15];
    (is_c ? Co : Bo)[row * 16 + (lane & 15)] = __float2bfloat16_rn(bc);
    if (dt_norm_w) {
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) ss_dt += __shfl_xor_sync(kFull, ss_dt, o);
        const float sc = rsqrtf(fmaf(ss_dt, 1.0f / static_cast<float>(R), eps));
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j < J) dt_low[row * R + lane + 32 * j] = __float2bfloat16_rn(v[j] * sc * dt_norm_w[lane + 32 * j]);
        // rows wider than 8 x 32 are summed again for the scaled store
        for (int j = 8; j < J; ++j)
            dt_low[row * R + lane + 32 * j] = __float2bfloat16_rn(col_sum(j) * sc * dt_norm_w[lane + 32 * j]);
    }
}

// Sum of `splits` fp32 partial products ([splits][n] floats, n a multiple of
// 4) into fp32 or bf16 output: four elements per thread.
template <bool OUT_BF16>
__global__ void __launch_bounds__(256)
splitk_reduce_kernel(const float* __restrict__ part, int splits, int64_t n, void* __restrict__ out)
{
    const int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
    if (i >= n) return;
    float4 acc = *reinterpret_cast<const float4*>(part + i);
    for (int s = 1; s < splits; ++s) {
        const float4 v = *reinterpret_cast<const float4*>(part + s * n + i);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    if constexpr (OUT_BF16) {
        uint2 w;
        w.x = pack_bf16x2(acc.x, acc.y);
        w.y = pack_bf16x2(acc.z, acc.w);
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out) + i) = w;
    } else {
        *reinterpret_cast<float4*>(static_cast<float*>(out) + i) = acc;
    }
}

}  // namespace mm
