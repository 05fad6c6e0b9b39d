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
// Work decomposition: one thread per (layer, batch, channel) row.  A warp
// covers 32 consecutive channels of one (layer, batch): its 16-float state
// rows form one contiguous 2 KB span, its 3-element conv windows one
// contiguous span, and B/C of the (layer, batch) are the same for every lane
// (one broadcast load).  Per row the kernel moves 64 B of state in and out,
// 3 window values in and out, x/z/dt in and y out: the whole step is a single
// streaming pass over HBM, with the 16 exponentials per row on the MUFU pipe
// well under the memory time.
#pragma once

#include "mixer_common.cuh"

namespace mm {

template <typename T, typename M>
__global__ void __launch_bounds__(256)
state_update_kernel(const T* __restrict__ x, const T* __restrict__ z, const T* __restrict__ dt,
                    const float* __restrict__ conv_w, const float* __restrict__ conv_b,
                    const float* __restrict__ dt_bias, const float* __restrict__ Dskip,
                    const float* __restrict__ A, const T* __restrict__ Bm, const T* __restrict__ Cm,
                    float* __restrict__ ssm_state, T* __restrict__ conv_state, T* __restrict__ y,
                    int64_t rows, int batch, int D)
{
    const int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    const int64_t lb = r / D;                 // layer * batch + b
    const int d = static_cast<int>(r - lb * D);
    const int64_t layer = lb / batch;
    const int64_t ld = layer * D + d;         // parameter row

    // ---- parameters of (layer, d)
    const float4 w = *reinterpret_cast<const float4*>(conv_w + ld * 4);
    const float cb = conv_b ? conv_b[ld] : 0.0f;
    const float bias = dt_bias[ld];
    const float dsk = Dskip ? Dskip[ld] : 0.0f;

    // ---- token inputs and window
    T* cs = conv_state + r * 3;
    const T w0raw = cs[0], w1raw = cs[1], w2raw = cs[2];
    const float c0 = Act<T>::to_f32(w0raw), c1 = Act<T>::to_f32(w1raw), c2 = Act<T>::to_f32(w2raw);
    const T xraw = x[r];
    const float xv = Act<T>::to_f32(xraw);
    const float zv = Act<T>::load(z + r);
    const float dtv = Act<T>::load(dt + r);

    float pre = fmaf(w.x, c0, cb);
    pre = fmaf(w.y, c1, pre);
    pre = fmaf(w.z, c2, pre);
    pre = fmaf(w.w, xv, pre);
    const float u = M::silu(pre);

    float l;
    if constexpr (M::step_scale == 1.0f) l = M::step(dtv, bias);
    else l = M::step2(dtv, bias * kLog2e);
    const float s = l * M::step_scale * u;    // Delta * u

    // ---- B, C of (layer, b): 16 each
    float bv[16], cv[16];
    if constexpr (sizeof(T) == 2) {
        const uint4* bp = reinterpret_cast<const uint4*>(Bm + lb * 16);
        const uint4* cp = reinterpret_cast<const uint4*>(Cm + lb * 16);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const uint4 bb = bp[q], cc = cp[q];
            const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
            const uint32_t cw[4] = {cc.x, cc.y, cc.z, cc.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                bv[q * 8 + 2 * k] = __uint_as_float(bw[k] << 16);
                bv[q * 8 + 2 * k + 1] = __uint_as_float(bw[k] & 0xffff0000u);
                cv[q * 8 + 2 * k] = __uint_as_float(cw[k] << 16);
                cv[q * 8 + 2 * k + 1] = __uint_as_float(cw[k] & 0xffff0000u);
            }
        }
    } else {
        const float4* bp = reinterpret_cast<const float4*>(Bm + lb * 16);
        const float4* cp = reinterpret_cast<const float4*>(Cm + lb * 16);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 bb = bp[q], cc = cp[q];
            bv[4 * q] = bb.x; bv[4 * q + 1] = bb.y; bv[4 * q + 2] = bb.z; bv[4 * q + 3] = bb.w;
            cv[4 * q] = cc.x; cv[4 * q + 1] = cc.y; cv[4 * q + 2] = cc.z; cv[4 * q + 3] = cc.w;
        }
    }

    // ---- state update and readout
    float4* hp = reinterpret_cast<float4*>(ssm_state + r * 16);
    const float4* ap = reinterpret_cast<const float4*>(A + ld * 16);
    float acc = 0.0f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float4 h = hp[q];
        const float4 a = ap[q];
        h.x = fmaf(M::decay(l, a.x), h.x, s * bv[4 * q + 0]);
        h.y = fmaf(M::decay(l, a.y), h.y, s * bv[4 * q + 1]);
        h.z = fmaf(M::decay(l, a.z), h.z, s * bv[4 * q + 2]);
        h.w = fmaf(M::decay(l, a.w), h.w, s * bv[4 * q + 3]);
        acc = fmaf(cv[4 * q + 0], h.x, acc);
        acc = fmaf(cv[4 * q + 1], h.y, acc);
        acc = fmaf(cv[4 * q + 2], h.z, acc);
        acc = fmaf(cv[4 * q + 3], h.w, acc);
        hp[q] = h;
    }
    const float yv = fmaf(dsk, u, acc) * M::silu(zv);
    y[r] = Act<T>::from_f32(yv);

    // ---- slide the window: drop the oldest, append this token's raw x
    cs[0] = w1raw;
    cs[1] = w2raw;
    cs[2] = xraw;
}

}  // namespace mm
