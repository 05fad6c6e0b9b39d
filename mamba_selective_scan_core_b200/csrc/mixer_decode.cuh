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
// out; the per-layer parameters and B/C are shared and stay in L2.
//
// Work decomposition, chosen so every global access of a warp is one
// contiguous span and the shared per-layer data is read once per warp:
//   * a warp owns one layer's block of 32 channels and walks a chunk of 16
//     batch rows for it; A and the per-channel parameters are read from
//     HBM/L2 once and from L1 for the other rows (A is not held in registers:
//     that would cost 16 of them and force spills or lower occupancy);
//   * in the row phase lane i does the per-row work of channel i (window, conv,
//     SiLU, softplus, SiLU(z)) with coalesced 2-byte accesses;
//   * in four state passes, pass p covers rows 8p..8p+7 with 4 lanes per row
//     and 4 states per lane, so the warp's 16-byte state and A accesses form
//     one contiguous 512-byte span; (Delta, Delta*u) arrive from the row's
//     lane by shuffle and the partial readouts go back the same way.
// State loads and stores are marked streaming (evict-first) so the
// parameters, reused by every batch row, stay in L2.
#pragma once

#include "mixer_common.cuh"

#ifndef MM_DECODE_MIN_BLOCKS
#define MM_DECODE_MIN_BLOCKS 4     // CTAs of 256 threads per SM: 64 registers, no spills
#endif

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

// RMSNorm of a 16-entry row held as 4 values in each lane of a quad: the
// sum of squares is combined across the quad by two shuffles.
__device__ __forceinline__ float4 rms_scale4(float4 v, const float* w, float eps) {
    float ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, v.w * v.w)));
    ss += __shfl_xor_sync(kFull, ss, 1);
    ss += __shfl_xor_sync(kFull, ss, 2);
    const float sc = rsqrtf(fmaf(ss, 1.0f / 16.0f, eps));
    const float4 wv = __ldg(reinterpret_cast<const float4*>(w));
    return make_float4(v.x * sc * wv.x, v.y * sc * wv.y, v.z * sc * wv.z, v.w * sc * wv.w);
}

// Batch rows a warp walks for one (layer, 32-channel block).  A and the
// per-channel parameters come from HBM/L2 once per warp and from L1 for the
// other rows, so the per-layer data costs 1/16 of a row's traffic.
constexpr int kDecodeBatchChunk = 16;

// The fp32 path's libm calls need more registers; it keeps 3 CTAs per SM.
// NORM: the RMSNorm of each row's B and C is applied (a separate instance at 3
// CTAs per SM, so the plain step keeps its register budget and occupancy).
template <typename T, typename M, bool NORM>
__global__ void __launch_bounds__(256, (sizeof(T) == 4 || NORM) ? 3 : MM_DECODE_MIN_BLOCKS)
state_update_kernel(const T* __restrict__ x, const T* __restrict__ z, const T* __restrict__ dt,
                    const float* __restrict__ conv_w, const float* __restrict__ conv_b,
                    const float* __restrict__ dt_bias, const float* __restrict__ Dskip,
                    const float* __restrict__ A, const T* __restrict__ Bm, const T* __restrict__ Cm,
                    float* __restrict__ ssm_state, T* __restrict__ conv_state, T* __restrict__ y,
                    int n_layers, int batch, int D,
                    const float* __restrict__ b_norm_w, const float* __restrict__ c_norm_w, float norm_eps)
{
    const int lane = threadIdx.x & 31;
    const int q = lane & 3;            // which 4 states of a row
    const int rr = lane >> 2;          // row within a pass
    const int cblocks = (D + 31) / 32;
    const int bchunks = (batch + kDecodeBatchChunk - 1) / kDecodeBatchChunk;
    const int64_t warp = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (warp >= static_cast<int64_t>(n_layers) * cblocks * bchunks) return;
    const int bc = static_cast<int>(warp % bchunks);
    const int cb = static_cast<int>((warp / bchunks) % cblocks);
    const int layer = static_cast<int>(warp / (static_cast<int64_t>(bchunks) * cblocks));
    const int d0 = cb * 32;
    const int b_begin = bc * kDecodeBatchChunk;
    const int b_end = min(batch, b_begin + kDecodeBatchChunk);
    // index checks of the checked build (all `true` in the release build); the
    // decode has no status word, so a skipped access shows in the fault word
    const int64_t nLD = static_cast<int64_t>(n_layers) * D, nLB = static_cast<int64_t>(n_layers) * batch;
    const int64_t nLBD = nLB * D;
    auto inb = [&](int64_t first, int64_t count, int64_t extent) {
        return mm_in_bounds(first, count, extent, nullptr, 0ull);
    };

    // ---- per-(layer, channel) values shared by every batch row
    const float* Aw = A + (static_cast<int64_t>(layer) * D + d0 + rr) * 16 + q * 4;  // pass 0's slice
    const int dl = d0 + lane;          // this lane's channel in the row phase
    const bool lok = dl < D;
    float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
    float cbias = 0.f, bias2 = 0.f, dsk = 0.f;
    if (lok && inb((static_cast<int64_t>(layer) * D + dl) * 4, 4, nLD * 4) &&
        inb(static_cast<int64_t>(layer) * D + dl, 1, nLD)) {
        const int64_t ld = static_cast<int64_t>(layer) * D + dl;
        w = *reinterpret_cast<const float4*>(conv_w + ld * 4);
        cbias = conv_b ? conv_b[ld] : 0.0f;
        bias2 = dt_bias[ld];
        if constexpr (M::step_scale != 1.0f) bias2 *= kLog2e;
        dsk = Dskip ? Dskip[ld] : 0.0f;
    }

#pragma unroll 1
    for (int b = b_begin; b < b_end; ++b) {
        const int64_t lb = static_cast<int64_t>(layer) * batch + b;
        const int64_t rowbase = lb * D + d0;
        // the row's whole 2 KB of state first, so it is in flight during the row phase
        float4 hv[4];
#pragma unroll
        for (int pass = 0; pass < 4; ++pass)
            hv[pass] = d0 + pass * 8 + rr < D && inb((rowbase + pass * 8 + rr) * 16 + q * 4, 4, nLBD * 16)
                           ? __ldcs(reinterpret_cast<const float4*>(ssm_state + (rowbase + pass * 8 + rr) * 16 + q * 4))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        const bool bcok = inb(lb * 16 + q * 4, 4, nLB * 16);
        float4 bq = bcok ? Vec4Act<T>::load(Bm + lb * 16 + q * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
        float4 cq = bcok ? Vec4Act<T>::load(Cm + lb * 16 + q * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
        // optional RMSNorm of the row's B and C over their 16 entries (4 lanes x 4)
        if constexpr (NORM) {
            if (b_norm_w) bq = rms_scale4(bq, b_norm_w + static_cast<int64_t>(layer) * 16 + q * 4, norm_eps);
            if (c_norm_w) cq = rms_scale4(cq, c_norm_w + static_cast<int64_t>(layer) * 16 + q * 4, norm_eps);
        }

        // ---- row phase: lane i does the per-row work of channel d0 + i
        float l = 0.f, s = 0.f, u = 0.f, gz = 0.f;
        const bool rok = lok && inb((rowbase + lane) * 3, 3, nLBD * 3) && inb(rowbase + lane, 1, nLBD);
        if (rok) {
            const int64_t r = rowbase + lane;
            T* cs = conv_state + r * 3;
            const T w0 = cs[0], w1 = cs[1], w2 = cs[2];
            const T xr = x[r];
            const float dtv = Act<T>::load(dt + r);
            const float zv = Act<T>::load(z + r);
            float pre = fmaf(w.x, Act<T>::to_f32(w0), cbias);
            pre = fmaf(w.y, Act<T>::to_f32(w1), pre);
            pre = fmaf(w.z, Act<T>::to_f32(w2), pre);
            pre = fmaf(w.w, Act<T>::to_f32(xr), pre);
            u = M::silu(pre);
            if constexpr (M::step_scale == 1.0f) l = M::step(dtv, bias2);
            else l = M::step2(dtv, bias2);
            s = l * M::step_scale * u;                  // Delta * u
            gz = M::silu(zv);
            // slide the window: drop the oldest, append this token's raw x
            cs[0] = w1;
            cs[1] = w2;
            cs[2] = xr;
        }

        // ---- state passes: 4 lanes per row, 4 states per lane
        float ysum = 0.f;              // lane i ends with channel d0 + i's readout
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
            const int src = pass * 8 + rr;              // lane holding this row's per-row values
            const float lr = __shfl_sync(kFull, l, src);
            const float sr = __shfl_sync(kFull, s, src);
            float part = 0.f;
            if (d0 + src < D && inb((static_cast<int64_t>(layer) * D + d0 + src) * 16 + q * 4, 4, nLD * 16) &&
                inb((rowbase + src) * 16 + q * 4, 4, nLBD * 16)) {
                float4 h = hv[pass];
                const float4 a = __ldg(reinterpret_cast<const float4*>(Aw + pass * 8 * 16));  // L1 after row 0
                h.x = fmaf(M::decay(lr, a.x), h.x, sr * bq.x);
                h.y = fmaf(M::decay(lr, a.y), h.y, sr * bq.y);
                h.z = fmaf(M::decay(lr, a.z), h.z, sr * bq.z);
                h.w = fmaf(M::decay(lr, a.w), h.w, sr * bq.w);
                __stcs(reinterpret_cast<float4*>(ssm_state + (rowbase + src) * 16 + q * 4), h);
                part = fmaf(cq.x, h.x, fmaf(cq.y, h.y, fmaf(cq.z, h.z, cq.w * h.w)));
            }
            part += __shfl_xor_sync(kFull, part, 1);
            part += __shfl_xor_sync(kFull, part, 2);
            // every lane of the quad now holds row src's readout; lane src takes it
            const float got = __shfl_sync(kFull, part, ((lane - pass * 8) & 7) * 4);
            if ((lane >> 3) == pass) ysum = got;
        }
        if (rok) y[rowbase + lane] = Act<T>::from_f32(fmaf(dsk, u, ysum) * gz);
    }
}

}  // namespace mm
