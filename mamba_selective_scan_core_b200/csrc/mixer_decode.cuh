// One-token state update (decode) of the Mamba mixer core for a stack of
// independent layers.
//
// The step is the forward's body for a single token (Jamba hybrid
// SSM-Transformer lesson, "SSM in one page": y_t needs only h_{t-1} and x_t):
//   window = [cs0, cs1, cs2, x]              (raw x, oldest first)
//   u      = SiLU(conv_b + sum_k conv_w[k] * window[k])
//   Delta  = softplus(dt + dt_bias)
//   h[n]   = exp(Delta * A[n]) * h[n] + Delta * B[n] * u
//   y      = (sum_n C[n] h[n] + Dskip * u) * SiLU(z)
//   window = [cs1, cs2, x]
//
// It is a single streaming pass over HBM: per (layer, batch, channel) row,
// 64 B of state in and out, the 3-value window in and out, x/z/dt in and y
// out.  Work decomposition, chosen so every global access of a warp is one
// contiguous span:
//   * a warp owns 32 consecutive rows; in the row phase lane i does the
//     per-row work of row i (window, conv, SiLU, softplus, SiLU(z)) with
//     coalesced 2-byte accesses;
//   * in four state passes, pass p covers rows 8p..8p+7 with 4 lanes per row
//     and 4 states per lane, so the warp's 16-byte state and A accesses form
//     one contiguous 512-byte span; (Delta, Delta*u) arrive from the row's
//     lane by shuffle and the partial readouts go back the same way.
// State loads and stores are marked streaming (evict-first) so the per-layer
// parameters, reused by every batch row, stay in L2.
#pragma once

#include "mixer_common.cuh"

namespace mm {

template <typename T> struct Vec4Act;
template <> struct Vec4Act<float> {
    __device__ __forceinline__ static float4 load(const float* p) { return *reinterpret_cast<const float4*>(p); }
};
template <> struct Vec4Act<__nv_bfloat16> {
    __device__ __forceinline__ static float4 load(const __nv_bfloat16* p) {
        const uint2 v = *reinterpret_cast<const uint2*>(p);
        return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                           __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
    }
};

template <typename T, typename M>
__global__ void __launch_bounds__(256)
state_update_kernel(const T* __restrict__ x, const T* __restrict__ z, const T* __restrict__ dt,
                    const float* __restrict__ conv_w, const float* __restrict__ conv_b,
                    const float* __restrict__ dt_bias, const float* __restrict__ Dskip,
                    const float* __restrict__ A, const T* __restrict__ Bm, const T* __restrict__ Cm,
                    float* __restrict__ ssm_state, T* __restrict__ conv_state, T* __restrict__ y,
                    int64_t rows, int batch, int D)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp_row0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31));
    if (warp_row0 >= rows) return;                      // whole warp past the end

    // ---------------------------------------------------------- row phase
    const int64_t r = warp_row0 + lane;
    const bool live = r < rows;
    float l = 0.f, s = 0.f, u = 0.f, gz = 0.f, dsk = 0.f;
    if (live) {
        const int64_t lb = r / D;
        const int d = static_cast<int>(r - lb * D);
        const int64_t ld = (lb / batch) * D + d;       // parameter row (layer, d)
        const float4 w = *reinterpret_cast<const float4*>(conv_w + ld * 4);
        const float cb = conv_b ? conv_b[ld] : 0.0f;
        const float bias = dt_bias[ld];
        dsk = Dskip ? Dskip[ld] : 0.0f;
        T* cs = conv_state + r * 3;
        const T c0 = cs[0], c1 = cs[1], c2 = cs[2];
        const T xr = x[r];
        float pre = fmaf(w.x, Act<T>::to_f32(c0), cb);
        pre = fmaf(w.y, Act<T>::to_f32(c1), pre);
        pre = fmaf(w.z, Act<T>::to_f32(c2), pre);
        pre = fmaf(w.w, Act<T>::to_f32(xr), pre);
        u = M::silu(pre);
        const float dtv = Act<T>::load(dt + r);
        if constexpr (M::step_scale == 1.0f) l = M::step(dtv, bias);
        else l = M::step2(dtv, bias * kLog2e);
        s = l * M::step_scale * u;                      // Delta * u
        gz = M::silu(Act<T>::load(z + r));
        // slide the window: drop the oldest, append this token's raw x
        cs[0] = c1;
        cs[1] = c2;
        cs[2] = xr;
    }

    // ---------------------------------------------------------- state passes
    const int q = lane & 3;            // which 4 states of the row
    const int rr = lane >> 2;          // row within the pass
    float ysum = 0.f;                  // lane i ends with row i's readout
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
        const int src = pass * 8 + rr;                  // lane holding this row's per-row values
        const float lr = __shfl_sync(kFull, l, src);
        const float sr = __shfl_sync(kFull, s, src);
        const int64_t row = warp_row0 + src;
        float part = 0.f;
        if (row < rows) {
            const int64_t lb = row / D;
            const int d = static_cast<int>(row - lb * D);
            const int64_t ld = (lb / batch) * D + d;
            float4* hp = reinterpret_cast<float4*>(ssm_state + row * 16 + q * 4);
            float4 h = __ldcs(hp);
            const float4 a = *reinterpret_cast<const float4*>(A + ld * 16 + q * 4);
            const float4 bv = Vec4Act<T>::load(Bm + lb * 16 + q * 4);
            const float4 cv = Vec4Act<T>::load(Cm + lb * 16 + q * 4);
            h.x = fmaf(M::decay(lr, a.x), h.x, sr * bv.x);
            h.y = fmaf(M::decay(lr, a.y), h.y, sr * bv.y);
            h.z = fmaf(M::decay(lr, a.z), h.z, sr * bv.z);
            h.w = fmaf(M::decay(lr, a.w), h.w, sr * bv.w);
            __stcs(hp, h);
            part = fmaf(cv.x, h.x, fmaf(cv.y, h.y, fmaf(cv.z, h.z, cv.w * h.w)));
        }
        part += __shfl_xor_sync(kFull, part, 1);
        part += __shfl_xor_sync(kFull, part, 2);
        // every lane of the quad now holds row src's readout; lane src takes it
        const float got = __shfl_sync(kFull, part, ((lane - pass * 8) & 7) * 4);
        if ((lane >> 3) == pass) ysum = got;
    }
    if (live) y[r] = Act<T>::from_f32(fmaf(dsk, u, ysum) * gz);
}

}  // namespace mm
