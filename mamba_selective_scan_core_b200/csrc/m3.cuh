// The Mamba-3 form of the selective scan: the lesson's "Mamba-3" section
// names its three changes over Mamba-2 -- an exponential-trapezoidal
// discretisation whose conv-like two-tap rule acts on the state input inside
// the recurrence, a complex-valued state (equivalently a data-dependent
// rotary embedding of the state), and multi-input multi-output projections.
// Per head h, channel c, and state pair k (entries 2k, 2k+1 = real and
// imaginary part):
//
//     a_t[k] = exp(Delta_t A[h]) (cos(Delta_t theta[h,k]) + i sin(Delta_t theta[h,k]))
//     u_t[k] = sum_r (B_t[r,2k] + i B_t[r,2k+1]) x_t[r,c]
//     s_t[k] = a_t[k] (s_{t-1}[k] + (1 - lambda_t) Delta_t u_{t-1}[k]) + lambda_t Delta_t u_t[k]
//     y_t[r,c] = (sum_k Re(conj(C_t[r,k]) s_t[k]) + D[h] x_t[r,c]) SiLU(z_t[r,c])
//
// d_state 16 (8 complex pairs): a channel's state lives in one thread's
// registers, in fp32.  The recurrence is linear in the state, so a sequence
// is cut into time chunks for parallelism, an exact regrouping:
//   m3_chunk_kernel<false> (summary pass, chunks 0..K-2): each chunk's end
//       state from a zero start (the first token's trapezoid tap on the
//       previous token's input included), per channel, and the chunk's
//       product of a_t, per head;
//   m3_chunk_kernel<true> (full pass, every chunk): the entering state as
//       h0 carried through the earlier chunks' (product, end state) pairs,
//       then the recurrence with readout, skip and gate; the last chunk
//       writes h_last.
// Per-(token, head) factors -- a_t (one exp and one sincos per pair) and the
// two tap weights -- are computed once per CTA tile into shared memory, as
// are the tile's B and C rows; x, z and y move per thread, 2 bytes each, a
// warp's 32 channels contiguous.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "mixer_common.cuh"

namespace mm {

constexpr int kM3Pairs = 8;        // d_state 16 = 8 complex pairs
constexpr int kM3N = 2 * kM3Pairs;
constexpr int kM3P = 64;           // channels per head
constexpr int kM3Threads = 128;    // channels per CTA: two heads
constexpr int kM3Heads = kM3Threads / kM3P;
constexpr int kM3Tile = 32;        // tokens per staged tile
constexpr int kM3MaxRank = 4;

struct M3Params {
    const __nv_bfloat16* x;        // [B][L][R][H*P]
    const __nv_bfloat16* z;        // [B][L][R][H*P] or null
    const __nv_bfloat16* dt;       // [B][L][H]
    const __nv_bfloat16* trap;     // [B][L][H] or null (1/2)
    const float* dt_bias;          // [H] or null
    const float* A;                // [H]
    const float* theta;            // [H][N/2]
    const __nv_bfloat16* Bm;       // [B][L][R][G][N]
    const __nv_bfloat16* Cm;       // [B][L][R][G][N]
    const float* Dskip;            // [H] or null
    const float* h0;               // [B][H][P][N] or null
    const __nv_bfloat16* x_prev;   // [B][R][H*P] or null
    const __nv_bfloat16* B_prev;   // [B][R][G][N] or null
    __nv_bfloat16* y;              // [B][L][R][H*P]
    float* h_last;                 // [B][H][P][N]
    float* ws_state;               // [K-1][B][H*P][N]   chunk end states from zero
    float* ws_prod;                // [K-1][B][H][N]     chunk products of a_t (pairs)
    int64_t L, chunk_len;
    int R, H, G, chunks;
};

struct M3Smem {
    float2 a[kM3Tile][kM3Heads][kM3Pairs];             // a_t per head and pair
    float2 w[kM3Tile][kM3Heads];                        // ((1 - lambda) Delta, lambda Delta)
    float4 b[kM3Tile][kM3MaxRank][kM3Heads][kM3N / 4];   // B rows of each head's group
    float4 c[kM3Tile][kM3MaxRank][kM3Heads][kM3N / 4];   // C rows
};

__device__ __forceinline__ float m3_bf(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// Thread j's channel input u of token t (or of the token before the call):
// sum_r (B[r, 2k] + i B[r, 2k+1]) x[r], from global rows.
__device__ __forceinline__ void m3_input_global(const M3Params& p, const __nv_bfloat16* xrow,
                                                const __nv_bfloat16* brow, int64_t x_rstride,
                                                int64_t b_rstride, float (&ur)[kM3Pairs], float (&ui)[kM3Pairs]) {
#pragma unroll
    for (int k = 0; k < kM3Pairs; ++k) ur[k] = ui[k] = 0.0f;
    for (int r = 0; r < p.R; ++r) {
        const float xv = m3_bf(xrow + r * x_rstride);
        const __nv_bfloat16* br = brow + r * b_rstride;
#pragma unroll
        for (int k = 0; k < kM3Pairs; ++k) {
            ur[k] = fmaf(m3_bf(br + 2 * k), xv, ur[k]);
            ui[k] = fmaf(m3_bf(br + 2 * k + 1), xv, ui[k]);
        }
    }
}

template <bool FULL>
__global__ void __launch_bounds__(kM3Threads)
m3_chunk_kernel(const M3Params p)
{
    __shared__ __align__(16) M3Smem sm;
    const int tid = threadIdx.x;
    const int64_t C = static_cast<int64_t>(p.H) * kM3P;
    const int64_t c = static_cast<int64_t>(blockIdx.x) * kM3Threads + tid;   // channel
    const int h0_ = blockIdx.x * kM3Heads;                                    // first head of the CTA
    const int hl = tid / kM3P;                                                // this thread's head, local
    const int h = h0_ + hl;
    const int chunk = blockIdx.y;
    const int b = blockIdx.z;
    const int64_t t0 = static_cast<int64_t>(chunk) * p.chunk_len;
    const int64_t t1 = min(p.L, t0 + p.chunk_len);
    const int R = p.R;
    const int64_t xr = C;                              // elements between the R inputs of a token
    const int64_t xt = static_cast<int64_t>(R) * C;    // ... between tokens
    const int64_t br = static_cast<int64_t>(p.G) * kM3N;
    const int64_t bt = static_cast<int64_t>(R) * br;
    const int g = h * p.G / p.H;

    // the state entering the chunk
    float sr[kM3Pairs], si[kM3Pairs];
#pragma unroll
    for (int k = 0; k < kM3Pairs; ++k) sr[k] = si[k] = 0.0f;
    if (FULL) {
        if (p.h0) {
            const float4* hp = reinterpret_cast<const float4*>(p.h0 + (static_cast<int64_t>(b) * C + c) * kM3N);
#pragma unroll
            for (int q = 0; q < kM3N / 4; ++q) {
                const float4 v = hp[q];
                sr[2 * q] = v.x; si[2 * q] = v.y; sr[2 * q + 1] = v.z; si[2 * q + 1] = v.w;
            }
        }
        // carried through the earlier chunks: s = prod_c' s + e_c'
        for (int cc = 0; cc < chunk; ++cc) {
            const float4* pp = reinterpret_cast<const float4*>(
                p.ws_prod + ((static_cast<int64_t>(cc) * gridDim.z + b) * p.H + h) * kM3N);
            const float4* ep = reinterpret_cast<const float4*>(
                p.ws_state + ((static_cast<int64_t>(cc) * gridDim.z + b) * C + c) * kM3N);
#pragma unroll
            for (int q = 0; q < kM3N / 4; ++q) {
                const float4 a = pp[q], e = ep[q];
                const int k0 = 2 * q, k1 = 2 * q + 1;
                float r0 = fmaf(a.x, sr[k0], fmaf(-a.y, si[k0], e.x));
                float i0 = fmaf(a.x, si[k0], fmaf(a.y, sr[k0], e.y));
                float r1 = fmaf(a.z, sr[k1], fmaf(-a.w, si[k1], e.z));
                float i1 = fmaf(a.z, si[k1], fmaf(a.w, sr[k1], e.w));
                sr[k0] = r0; si[k0] = i0; sr[k1] = r1; si[k1] = i1;
            }
        }
    }
    // the previous token's input u (the trapezoid's first tap)
    float ur[kM3Pairs], ui[kM3Pairs];
    if (t0 > 0) {
        const int64_t row = static_cast<int64_t>(b) * p.L + (t0 - 1);
        m3_input_global(p, p.x + row * xt + c, p.Bm + row * bt + g * kM3N, xr, br, ur, ui);
    } else if (p.x_prev && p.B_prev) {
        m3_input_global(p, p.x_prev + static_cast<int64_t>(b) * R * C + c,
                        p.B_prev + static_cast<int64_t>(b) * R * br + g * kM3N, xr, br, ur, ui);
    } else {
#pragma unroll
        for (int k = 0; k < kM3Pairs; ++k) ur[k] = ui[k] = 0.0f;
    }
    // the chunk's product of a_t (summary pass; the head's first thread keeps it)
    float pr[kM3Pairs], pi[kM3Pairs];
#pragma unroll
    for (int k = 0; k < kM3Pairs; ++k) { pr[k] = 1.0f; pi[k] = 0.0f; }

    const float dsk = p.Dskip ? p.Dskip[h] : 0.0f;
    for (int64_t ts = t0; ts < t1; ts += kM3Tile) {
        const int T = static_cast<int>(min(static_cast<int64_t>(kM3Tile), t1 - ts));
        __syncthreads();   // the previous tile's factors are consumed
        // factors of each (token, head): a_t per pair, then the tap weights
        for (int e = tid; e < kM3Tile * kM3Heads * kM3Pairs; e += kM3Threads) {
            const int k = e % kM3Pairs, hh = (e / kM3Pairs) % kM3Heads, tt = e / (kM3Pairs * kM3Heads);
            if (tt < T) {
                const int hd = h0_ + hh;
                const int64_t row = static_cast<int64_t>(b) * p.L + ts + tt;
                const float v = __bfloat162float(p.dt[row * p.H + hd]) + (p.dt_bias ? p.dt_bias[hd] : 0.0f);
                const float dl = fmaxf(v, 0.0f) + log1pf(expf(-fabsf(v)));
                const float mag = expf(dl * p.A[hd]);
                float sn, cs;
                sincosf(dl * p.theta[hd * kM3Pairs + k], &sn, &cs);
                sm.a[tt][hh][k] = make_float2(mag * cs, mag * sn);
                if (k == 0) {
                    const float lam = p.trap ? __bfloat162float(p.trap[row * p.H + hd]) : 0.5f;
                    sm.w[tt][hh] = make_float2((1.0f - lam) * dl, lam * dl);
                }
            }
        }
        // B and C rows of each head's group, widened to fp32
        for (int e = tid; e < kM3Tile * R * kM3Heads * (kM3N / 4); e += kM3Threads) {
            const int q = e % (kM3N / 4), hh = (e / (kM3N / 4)) % kM3Heads, r = (e / (kM3N / 4 * kM3Heads)) % R;
            const int tt = e / (kM3N / 4 * kM3Heads * R);
            if (tt < T) {
                const int gh = (h0_ + hh) * p.G / p.H;
                const int64_t off = (static_cast<int64_t>(b) * p.L + ts + tt) * bt + r * br + gh * kM3N + 4 * q;
                const uint2 bv = *reinterpret_cast<const uint2*>(p.Bm + off);
                const uint2 cv = *reinterpret_cast<const uint2*>(p.Cm + off);
                sm.b[tt][r][hh][q] = make_float4(__uint_as_float(bv.x << 16), __uint_as_float(bv.x & 0xffff0000u),
                                                 __uint_as_float(bv.y << 16), __uint_as_float(bv.y & 0xffff0000u));
                sm.c[tt][r][hh][q] = make_float4(__uint_as_float(cv.x << 16), __uint_as_float(cv.x & 0xffff0000u),
                                                 __uint_as_float(cv.y << 16), __uint_as_float(cv.y & 0xffff0000u));
            }
        }
        __syncthreads();

        for (int tt = 0; tt < T; ++tt) {
            const int64_t row = static_cast<int64_t>(b) * p.L + ts + tt;
            const __nv_bfloat16* xrow = p.x + row * xt + c;
            float xv[kM3MaxRank];
#pragma unroll
            for (int r = 0; r < kM3MaxRank; ++r) xv[r] = r < R ? m3_bf(xrow + r * xr) : 0.0f;
            // u_t
            float vr[kM3Pairs], vi[kM3Pairs];
#pragma unroll
            for (int k = 0; k < kM3Pairs; ++k) vr[k] = vi[k] = 0.0f;
#pragma unroll
            for (int r = 0; r < kM3MaxRank; ++r) {
                if (r < R) {
#pragma unroll
                    for (int q = 0; q < kM3N / 4; ++q) {
                        const float4 bb = sm.b[tt][r][hl][q];
                        vr[2 * q] = fmaf(bb.x, xv[r], vr[2 * q]);
                        vi[2 * q] = fmaf(bb.y, xv[r], vi[2 * q]);
                        vr[2 * q + 1] = fmaf(bb.z, xv[r], vr[2 * q + 1]);
                        vi[2 * q + 1] = fmaf(bb.w, xv[r], vi[2 * q + 1]);
                    }
                }
            }
            // s = a (s + (1 - lambda) Delta u_prev) + lambda Delta u
            const float2 w = sm.w[tt][hl];
#pragma unroll
            for (int k = 0; k < kM3Pairs; ++k) {
                const float2 a = sm.a[tt][hl][k];
                const float qr = fmaf(w.x, ur[k], sr[k]);
                const float qi = fmaf(w.x, ui[k], si[k]);
                sr[k] = fmaf(a.x, qr, fmaf(-a.y, qi, w.y * vr[k]));
                si[k] = fmaf(a.x, qi, fmaf(a.y, qr, w.y * vi[k]));
                ur[k] = vr[k];
                ui[k] = vi[k];
                if (!FULL) {
                    const float nr = a.x * pr[k] - a.y * pi[k];
                    pi[k] = a.x * pi[k] + a.y * pr[k];
                    pr[k] = nr;
                }
            }
            if (FULL) {
#pragma unroll
                for (int r = 0; r < kM3MaxRank; ++r) {
                    if (r < R) {
                        float acc = 0.0f;
#pragma unroll
                        for (int q = 0; q < kM3N / 4; ++q) {
                            const float4 cc = sm.c[tt][r][hl][q];
                            acc = fmaf(cc.x, sr[2 * q], acc);
                            acc = fmaf(cc.y, si[2 * q], acc);
                            acc = fmaf(cc.z, sr[2 * q + 1], acc);
                            acc = fmaf(cc.w, si[2 * q + 1], acc);
                        }
                        float yv = fmaf(dsk, xv[r], acc);
                        if (p.z) {
                            const float zv = m3_bf(p.z + row * xt + r * xr + c);
                            yv *= zv / (1.0f + expf(-zv));
                        }
                        p.y[row * xt + r * xr + c] = __float2bfloat16_rn(yv);
                    }
                }
            }
        }
    }

    if (FULL) {
        if (chunk == p.chunks - 1) {
            float4* hp = reinterpret_cast<float4*>(p.h_last + (static_cast<int64_t>(b) * C + c) * kM3N);
#pragma unroll
            for (int q = 0; q < kM3N / 4; ++q)
                hp[q] = make_float4(sr[2 * q], si[2 * q], sr[2 * q + 1], si[2 * q + 1]);
        }
    } else {
        float4* ep = reinterpret_cast<float4*>(
            p.ws_state + ((static_cast<int64_t>(chunk) * gridDim.z + b) * C + c) * kM3N);
#pragma unroll
        for (int q = 0; q < kM3N / 4; ++q) ep[q] = make_float4(sr[2 * q], si[2 * q], sr[2 * q + 1], si[2 * q + 1]);
        if (tid % kM3P == 0) {
            float4* pp = reinterpret_cast<float4*>(
                p.ws_prod + ((static_cast<int64_t>(chunk) * gridDim.z + b) * p.H + h) * kM3N);
#pragma unroll
            for (int q = 0; q < kM3N / 4; ++q) pp[q] = make_float4(pr[2 * q], pi[2 * q], pr[2 * q + 1], pi[2 * q + 1]);
        }
    }
}

}  // namespace mm
