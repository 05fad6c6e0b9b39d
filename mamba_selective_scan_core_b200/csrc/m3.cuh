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
//       pre-state (below) from a zero start, per channel, and the chunk's
//       product of a_t, per head;
//   m3_chunk_kernel<true> (full pass, every chunk): the entering pre-state
//       from h0 and the previous call's last input, carried through the
//       earlier chunks' (product, end pre-state) pairs, then the recurrence
//       with readout, skip and gate; the last chunk writes h_last.
// A CTA's tiles of x, z, B, C, dt and the trapezoid weight arrive by
// asynchronous 16-byte copies one tile ahead of the compute (two buffers).
// Per-(token, head) factors -- a_t (one exp and one sincos per pair) and the
// two tap weights -- are computed once per tile into shared memory, with the
// tile's B and C rows widened to fp32.  A thread holds two adjacent channels
// of one head (a warp per head), so every factor it reads serves both; y goes
// out as 4 bytes per thread, a warp's 64 channels contiguous.
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
constexpr int kM3Cpt = 2;          // channels per thread (adjacent, of one head)
constexpr int kM3Block = kM3Threads / kM3Cpt;   // threads per CTA: a warp per head
constexpr int kM3Tile = 32;        // chunk lengths are whole multiples of this
#ifndef MM_M3_TILE_ROWS
#define MM_M3_TILE_ROWS 16         // (token, input) rows per shared-memory tile: T = rows / R tokens
#endif
constexpr int kM3TileRows = MM_M3_TILE_ROWS;


static_assert(kM3Tile % kM3TileRows == 0, "tiles divide the chunks");

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
    unsigned long long* status;    // [1] <- the call's epoch (these kernels have no wait that can give up)
    unsigned long long status_epoch;
};

// Shared memory of a CTA: two buffers of raw tile inputs, filled by
// asynchronous copies one tile ahead of the compute, and the tile's
// per-(token, head) factors and widened B / C rows.  A tile is
// kM3TileRows / R tokens (R = 1, 2, 4), so its x and z rows are 4 KB each
// whatever R is.
struct M3Layout {
    int T, R;
    __host__ __device__ int xs() const { return T * R * kM3Threads * 2; }          // x or z rows, bf16
    __host__ __device__ int bs() const { return T * R * kM3Heads * kM3N * 2; }     // B or C rows, bf16
    __host__ __device__ int ds() const { return (T + 1) * kM3Heads * 2; }          // dt or trap (one token more), bf16
    __host__ __device__ int buf() const { return (2 * xs() + 2 * bs() + 2 * ds() + 15) & ~15; }
    __host__ __device__ int off_x(int i) const { return i * buf(); }
    __host__ __device__ int off_z(int i) const { return i * buf() + xs(); }
    __host__ __device__ int off_b(int i) const { return i * buf() + 2 * xs(); }
    __host__ __device__ int off_c(int i) const { return i * buf() + 2 * xs() + bs(); }
    __host__ __device__ int off_dt(int i) const { return i * buf() + 2 * xs() + 2 * bs(); }
    __host__ __device__ int off_tr(int i) const { return i * buf() + 2 * xs() + 2 * bs() + ds(); }
    __host__ __device__ int off_a() const { return 2 * buf(); }                      // float2 [T][heads][pairs]
    __host__ __device__ int off_w() const { return off_a() + T * kM3Heads * kM3Pairs * 8; }   // float2 [T+1][heads]
    __host__ __device__ int off_bf() const { return off_w() + (T + 1) * kM3Heads * 8; }       // float4 [T][R][heads][N/4]
    __host__ __device__ int off_cf() const { return off_bf() + T * R * kM3Heads * kM3N * 4; }
    __host__ __device__ int off_k() const { return off_cf() + T * R * kM3Heads * kM3N * 4; }  // float [T][heads][R][R]
    __host__ __device__ int bytes() const { return off_k() + T * kM3Heads * R * R * 4; }
};
__host__ __device__ inline M3Layout m3_layout(int R) { return M3Layout{kM3TileRows / R, R}; }

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" :: "r"(smem_addr(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" :: "r"(smem_addr(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
// wait until at most `pending` of this thread's committed groups are in flight
template <int pending>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" :: "n"(pending) : "memory"); }

__device__ __forceinline__ float m3_bf(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// sin and cos of an angle of any size: Cody and Waite's additive range
// reduction by 2 pi (a two-part constant: the float nearest 2 pi and the
// float nearest the rest), then the hardware approximations on [-pi, pi],
// whose absolute error there is about 2^-21.
__device__ __forceinline__ void m3_sincos(float x, float* sn, float* cs) {
    constexpr float kTwoPiHi = 6.28318548202514648f;       // float(2 pi)
    constexpr float kTwoPiLo = -1.7484555314695172e-07f;   // float(2 pi - kTwoPiHi)
    constexpr float kInvTwoPi = 0.15915494309189535f;
    const float k = rintf(x * kInvTwoPi);
    const float r = fmaf(-k, kTwoPiLo, fmaf(-k, kTwoPiHi, x));
    __sincosf(r, sn, cs);
}

// a * s + e for complex numbers held as (re, im) float2, on packed f32x2 operations:
// (a.re s.re - a.im s.im, a.re s.im + a.im s.re) + e
__device__ __forceinline__ float2 cmul_add(float2 a, float2 s, float2 e) {
    const float2 t = fma2(make_float2(-a.y, a.y), make_float2(s.y, s.x), e);
    return fma2(make_float2(a.x, a.x), s, t);
}
__device__ __forceinline__ float4 m3_widen4(uint2 v) {
    return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                       __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
}

// Thread j's channel input u of one token (or of the token before the call):
// sum_r (B[r, 2k] + i B[r, 2k+1]) x[r], from global rows, as (re, im) pairs.
template <int R>
__device__ __forceinline__ void m3_input_global(const __nv_bfloat16* xrow,
                                                const __nv_bfloat16* brow, int64_t x_rstride,
                                                int64_t b_rstride, float2 (&u)[kM3Pairs]) {
#pragma unroll
    for (int k = 0; k < kM3Pairs; ++k) u[k] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const float xv = m3_bf(xrow + r * x_rstride);
        const __nv_bfloat16* br = brow + r * b_rstride;
#pragma unroll
        for (int k = 0; k < kM3Pairs; ++k) {
            u[k].x = fmaf(m3_bf(br + 2 * k), xv, u[k].x);
            u[k].y = fmaf(m3_bf(br + 2 * k + 1), xv, u[k].y);
        }
    }
}

// Issue the asynchronous copies of one tile's raw inputs (tokens ts ..
// ts + n - 1 of sequence b) into buffer `buf`.
template <bool FULL, int R>
__device__ __forceinline__ void m3_issue_tile(const M3Params& p, const M3Layout& lay, unsigned char* sm, int buf,
                                              int b, int64_t ts, int n) {
    const int tid = threadIdx.x;
    const int64_t C = static_cast<int64_t>(p.H) * kM3P;
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kM3Threads;
    const int h0_ = blockIdx.x * kM3Heads;
    // x (and z): 16 pieces of 16 bytes per (token, input) row of the CTA's 128 channels
    for (int e = tid; e < n * R * 16; e += kM3Block) {
        const int q = e & 15, tr = e >> 4;                 // tr = token * R + r
        const int64_t g = (static_cast<int64_t>(b) * p.L + ts) * R * C + static_cast<int64_t>(tr) * C + c0 + 8 * q;
        cp_async16(sm + lay.off_x(buf) + tr * (kM3Threads * 2) + 16 * q, p.x + g);
        if (FULL && p.z) cp_async16(sm + lay.off_z(buf) + tr * (kM3Threads * 2) + 16 * q, p.z + g);
    }
    // B (and C) rows of each head's group: two 16-byte pieces per (token, input, head)
    const int64_t br = static_cast<int64_t>(p.G) * kM3N;
    for (int e = tid; e < n * R * kM3Heads * 2; e += kM3Block) {
        const int q = e & 1, hh = (e >> 1) % kM3Heads, tr = e / (2 * kM3Heads);
        const int gh = (h0_ + hh) * p.G / p.H;
        const int64_t g = ((static_cast<int64_t>(b) * p.L + ts) * R + tr) * br + gh * kM3N + 8 * q;
        const int so = (tr * kM3Heads + hh) * (kM3N * 2) + 16 * q;
        cp_async16(sm + lay.off_b(buf) + so, p.Bm + g);
        if (FULL) cp_async16(sm + lay.off_c(buf) + so, p.Cm + g);
    }
    // dt (and trap) of the CTA's two heads: 4 bytes per token, and of the
    // token after the tile when there is one (its trapezoid tap weight)
    const int nd = ts + n < p.L ? n + 1 : n;
    for (int e = tid; e < nd; e += kM3Block) {
        const int64_t g = (static_cast<int64_t>(b) * p.L + ts + e) * p.H + h0_;
        cp_async4(sm + lay.off_dt(buf) + 4 * e, p.dt + g);
        if (p.trap) cp_async4(sm + lay.off_tr(buf) + 4 * e, p.trap + g);
    }
}

// R: inputs per state (1, 2 or 4), a compile-time constant so that the
// per-token loops over inputs and outputs unroll.
template <bool FULL, int R>
__global__ void __launch_bounds__(kM3Block)
m3_chunk_kernel(const M3Params p)
{
    extern __shared__ __align__(16) unsigned char m3_sm[];
    constexpr int T = kM3TileRows / R;
    // tokens of the per-token loops unrolled together, so that one token's
    // shared-memory loads overlap another's arithmetic
    constexpr int kUnroll = R == 1 ? 4 : 2;
    if (FULL && p.status && threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
        p.status[1] = p.status_epoch;
    // the full pass, launched as a programmatic dependent of this summary
    // pass, may start its chunk-0 CTAs (which read no summary) at once
    if (!FULL) launch_dependents();
    const M3Layout lay = m3_layout(R);
    const int tid = threadIdx.x;
    const int cl = kM3Cpt * tid;                                              // first channel, CTA-local
    const int64_t C = static_cast<int64_t>(p.H) * kM3P;
    const int64_t c = static_cast<int64_t>(blockIdx.x) * kM3Threads + cl;    // first channel
    const int h0_ = blockIdx.x * kM3Heads;                                    // first head of the CTA
    const int hl = cl / kM3P;                                                 // this thread's head, local
    const int h = h0_ + hl;
    const int chunk = blockIdx.y;
    const int b = blockIdx.z;
    const int64_t t0 = static_cast<int64_t>(chunk) * p.chunk_len;
    const int64_t t1 = min(p.L, t0 + p.chunk_len);
    const int64_t xr = C;                              // elements between the R inputs of a token
    const int64_t xt = static_cast<int64_t>(R) * C;    // ... between tokens
    const int64_t br = static_cast<int64_t>(p.G) * kM3N;
    const int g = h * p.G / p.H;

    // the first tile's copies are in flight during the setup
    if (t0 < t1) m3_issue_tile<FULL, R>(p, lay, m3_sm, 0, b, t0, static_cast<int>(min(static_cast<int64_t>(T), t1 - t0)));
    cp_async_commit();

    // The kernel carries the pre-state  q_t = s_t + (1 - lambda_{t+1}) Delta_{t+1} u_t,
    // which obeys one multiply-add per pair and token,
    //     q_t = a_t q_{t-1} + omega_t u_t,   omega_t = lambda_t Delta_t + (1 - lambda_{t+1}) Delta_{t+1},
    // and reads out s_t = q_t - (1 - lambda_{t+1}) Delta_{t+1} u_t: the second
    // term is, per output r, sum_r' x_t[r'] (C_t[r] . B_t[r']) times that
    // weight, a per-(token, head) matrix kappa that also holds the skip D.
    // Past the last token the weight is 0, so q is s there.
    // A thread holds two adjacent channels of one head, so each per-token
    // factor it reads from shared memory serves both.  The state of pairs 2q
    // and 2q+1 of channel j as two packed registers: sre[j][q] their real
    // parts, sim[j][q] their imaginary parts, so that a complex multiply-add
    // of both pairs is four packed f32x2 FMAs with no operand swaps.  Memory
    // keeps (re, im) per pair.
    float2 sre[kM3Cpt][kM3Pairs / 2], sim[kM3Cpt][kM3Pairs / 2];
#pragma unroll
    for (int j = 0; j < kM3Cpt; ++j)
#pragma unroll
        for (int q = 0; q < kM3Pairs / 2; ++q) sre[j][q] = sim[j][q] = make_float2(0.0f, 0.0f);
    if (FULL) {
        // q_{-1} = h0 + (1 - lambda_0) Delta_0 u_{-1}
        if (p.h0) {
#pragma unroll
            for (int j = 0; j < kM3Cpt; ++j) {
                const float4* hp = reinterpret_cast<const float4*>(p.h0 + (static_cast<int64_t>(b) * C + c + j) * kM3N);
#pragma unroll
                for (int q = 0; q < kM3N / 4; ++q) {
                    const float4 v = hp[q];
                    sre[j][q] = make_float2(v.x, v.z);
                    sim[j][q] = make_float2(v.y, v.w);
                }
            }
        }
        if (p.x_prev && p.B_prev && p.L > 0) {
            const int64_t row = static_cast<int64_t>(b) * p.L;
            const float v = __bfloat162float(p.dt[row * p.H + h]) + (p.dt_bias ? p.dt_bias[h] : 0.0f);
            const float dl = fmaxf(v, 0.0f) + log1pf(expf(-fabsf(v)));
            const float lam = p.trap ? __bfloat162float(p.trap[row * p.H + h]) : 0.5f;
            const float2 w0 = make_float2((1.0f - lam) * dl, (1.0f - lam) * dl);
#pragma unroll
            for (int j = 0; j < kM3Cpt; ++j) {
                float2 up[kM3Pairs];
                m3_input_global<R>(p.x_prev + static_cast<int64_t>(b) * R * C + c + j,
                                p.B_prev + static_cast<int64_t>(b) * R * br + g * kM3N, xr, br, up);
#pragma unroll
                for (int q = 0; q < kM3Pairs / 2; ++q) {
                    sre[j][q] = fma2(w0, make_float2(up[2 * q].x, up[2 * q + 1].x), sre[j][q]);
                    sim[j][q] = fma2(w0, make_float2(up[2 * q].y, up[2 * q + 1].y), sim[j][q]);
                }
            }
        }
        // carried through the earlier chunks: q = prod_c' q + e_c' (their
        // summaries are complete and visible once the summary grid is)
        if (chunk > 0) grid_dependency_wait();
        for (int cc = 0; cc < chunk; ++cc) {
            const float4* pp = reinterpret_cast<const float4*>(
                p.ws_prod + ((static_cast<int64_t>(cc) * gridDim.z + b) * p.H + h) * kM3N);
            const float4* ep = reinterpret_cast<const float4*>(
                p.ws_state + ((static_cast<int64_t>(cc) * gridDim.z + b) * C + c) * kM3N);
#pragma unroll
            for (int q = 0; q < kM3N / 4; ++q) {
                const float4 a = pp[q];                // (re, im) of pairs 2q, 2q+1
                const float2 ar = make_float2(a.x, a.z), ai = make_float2(a.y, a.w);
#pragma unroll
                for (int j = 0; j < kM3Cpt; ++j) {
                    const float4 e = ep[j * (kM3N / 4) + q];
                    const float2 nr = fma2(ar, sre[j][q], fma2(make_float2(-ai.x, -ai.y), sim[j][q], make_float2(e.x, e.z)));
                    const float2 ni = fma2(ar, sim[j][q], fma2(ai, sre[j][q], make_float2(e.y, e.w)));
                    sre[j][q] = nr;
                    sim[j][q] = ni;
                }
            }
        }
    }
    // summary pass: the chunk's product of a_t for (head, pair) tid, tid < 16
    float2 prod = make_float2(1.0f, 0.0f);

    float2* fa = reinterpret_cast<float2*>(m3_sm + lay.off_a());
    float2* fw = reinterpret_cast<float2*>(m3_sm + lay.off_w());
    float4* fb = reinterpret_cast<float4*>(m3_sm + lay.off_bf());
    float4* fc = reinterpret_cast<float4*>(m3_sm + lay.off_cf());
    float* fk = reinterpret_cast<float*>(m3_sm + lay.off_k());
    // The per-tile factor loops below stride by the block size, a multiple of
    // heads x pairs, so each thread's elements there always belong to the same
    // head (and pair): its per-head parameters are loaded once, here.
    static_assert(kM3Block % (kM3Heads * kM3Pairs) == 0 && kM3Block % (kM3Heads * 16) == 0, "fixed head per thread");
    const int hw = h0_ + tid % kM3Heads;                              // tap weights
    const float bias_w = p.dt_bias ? p.dt_bias[hw] : 0.0f;
    const int ka = tid % kM3Pairs, ha = h0_ + (tid / kM3Pairs) % kM3Heads;   // a_t
    const float theta_a = p.theta[ha * kM3Pairs + ka];
    const float A_a = p.A[ha];
    const float dskip_k = p.Dskip ? p.Dskip[h0_ + (tid / (R * R)) % kM3Heads] : 0.0f;   // kappa
    int buf = 0;
    for (int64_t ts = t0; ts < t1; ts += T, buf ^= 1) {
        const int n = static_cast<int>(min(static_cast<int64_t>(T), t1 - ts));
        const int nd = ts + n < p.L ? n + 1 : n;
        // the next tile's copies go into the other buffer while this one is used
        const int64_t tn = ts + T;
        if (tn < t1) m3_issue_tile<FULL, R>(p, lay, m3_sm, buf ^ 1, b, tn, static_cast<int>(min(static_cast<int64_t>(T), t1 - tn)));
        cp_async_commit();
        cp_async_wait<1>();           // this tile's copies have landed (this thread's)
        __syncthreads();              // ... and every thread's
        const __nv_bfloat16* xs = reinterpret_cast<const __nv_bfloat16*>(m3_sm + lay.off_x(buf));
        const __nv_bfloat16* zs = reinterpret_cast<const __nv_bfloat16*>(m3_sm + lay.off_z(buf));
        const __nv_bfloat16* dts = reinterpret_cast<const __nv_bfloat16*>(m3_sm + lay.off_dt(buf));
        const __nv_bfloat16* trs = reinterpret_cast<const __nv_bfloat16*>(m3_sm + lay.off_tr(buf));
        // tap weights ((1 - lambda) Delta, lambda Delta) per (token, head), the
        // token after the tile included (zero past the sequence)
        for (int e = tid; e < (T + 1) * kM3Heads; e += kM3Block) {
            const int tt = e / kM3Heads;
            float2 w = make_float2(0.0f, 0.0f);
            if (tt < nd) {
                const float v = __bfloat162float(dts[e]) + bias_w;
                const float dl = fmaxf(v, 0.0f) + log1pf(expf(-fabsf(v)));
                const float lam = p.trap ? __bfloat162float(trs[e]) : 0.5f;
                w = make_float2((1.0f - lam) * dl, lam * dl);
            }
            fw[e] = w;
        }
        __syncthreads();
        // a_t per pair
        for (int e = tid; e < n * kM3Heads * kM3Pairs; e += kM3Block) {
            const int k = ka, th = e / kM3Pairs;
            const float2 w = fw[th];
            const float dl = w.x + w.y;
            float sn, cs;
            m3_sincos(dl * theta_a, &sn, &cs);
            const float mag = ex2_fast(dl * A_a * kLog2e);
            // per (token, head) and pair block q: (re 2q, re 2q+1, im 2q, im 2q+1)
            float* fq = reinterpret_cast<float*>(fa) + th * kM3N + (k >> 1) * 4 + (k & 1);
            fq[0] = mag * cs;
            fq[2] = mag * sn;
        }
        // omega_t B_t and C_t, widened to fp32
        const uint2* braw = reinterpret_cast<const uint2*>(m3_sm + lay.off_b(buf));
        const uint2* craw = reinterpret_cast<const uint2*>(m3_sm + lay.off_c(buf));
        for (int e = tid; e < n * R * kM3Heads * (kM3N / 4); e += kM3Block) {
            const int hh = (e / (kM3N / 4)) % kM3Heads, tt = e / (kM3N / 4 * kM3Heads * R);
            const float om = fw[tt * kM3Heads + hh].y + fw[(tt + 1) * kM3Heads + hh].x;
            const float4 bv = m3_widen4(braw[e]);      // (re, im, re, im) of pairs 2q, 2q+1
            fb[e] = make_float4(om * bv.x, om * bv.z, om * bv.y, om * bv.w);
            if (FULL) {
                const float4 cv = m3_widen4(craw[e]);
                fc[e] = make_float4(cv.x, cv.z, cv.y, cv.w);
            }
        }
        // kappa[t][head][r][r'] = D [r == r'] - (1 - lambda_{t+1}) Delta_{t+1} (C_t[r] . B_t[r'])
        if (FULL) {
            for (int e = tid; e < n * kM3Heads * R * R; e += kM3Block) {
                const int rp = e % R, r = (e / R) % R, hh = (e / (R * R)) % kM3Heads, tt = e / (R * R * kM3Heads);
                const uint2* bq = braw + ((tt * R + rp) * kM3Heads + hh) * (kM3N / 4);
                const uint2* cq = craw + ((tt * R + r) * kM3Heads + hh) * (kM3N / 4);
                float dot = 0.0f;
#pragma unroll
                for (int q = 0; q < kM3N / 4; ++q) {
                    const float4 bv = m3_widen4(bq[q]), cv = m3_widen4(cq[q]);
                    dot = fmaf(cv.x, bv.x, fmaf(cv.y, bv.y, fmaf(cv.z, bv.z, fmaf(cv.w, bv.w, dot))));
                }
                fk[e] = (r == rp ? dskip_k : 0.0f) - fw[(tt + 1) * kM3Heads + hh].x * dot;
            }
        }
        __syncthreads();
        if (!FULL) {
            // The summary pass needs only the chunk's end pre-state,
            //     F = sum_t (prod_{s>t} a_s) omega_t sum_r b_{t,r} x_{t,r},
            // whose factor V_{t,r} = (prod_{s>t} a_s) omega_t b_{t,r} is the
            // same for all channels of a head.  Within the tile: W_t = the
            // product of a_s over the tile's later tokens (16 threads, one per
            // (head, pair), walking back), P = the tile's whole product; then
            // V = W omega b in place of omega b.  Each channel then carries
            // F <- P F + sum_t x_t V_t.
            float* fW = reinterpret_cast<float*>(fc);           // [T][heads][N], split layout as fa
            float* fP = fk;                                       // [heads][N]
            if (tid < kM3Heads * kM3Pairs) {
                const int off = (tid / kM3Pairs) * kM3N + ((tid % kM3Pairs) >> 1) * 4 + (tid & 1);
                const float* faf = reinterpret_cast<const float*>(fa);
                float2 w = make_float2(1.0f, 0.0f);
                for (int tt = n - 1; tt >= 0; --tt) {
                    fW[tt * kM3Heads * kM3N + off] = w.x;
                    fW[tt * kM3Heads * kM3N + off + 2] = w.y;
                    w = cmul_add(make_float2(faf[tt * kM3Heads * kM3N + off], faf[tt * kM3Heads * kM3N + off + 2]), w,
                                 make_float2(0.0f, 0.0f));
                }
                fP[off] = w.x;
                fP[off + 2] = w.y;
                prod = cmul_add(w, prod, make_float2(0.0f, 0.0f));
            }
            __syncthreads();
            for (int e = tid; e < n * R * kM3Heads * (kM3N / 4); e += kM3Block) {
                const int q = e % (kM3N / 4), hh = (e / (kM3N / 4)) % kM3Heads, tt = e / (kM3N / 4 * kM3Heads * R);
                const float4 w = reinterpret_cast<const float4*>(fW)[(tt * kM3Heads + hh) * (kM3N / 4) + q];
                const float4 v = fb[e];     // (re, re, im, im) of pairs 2q, 2q+1
                fb[e] = make_float4(w.x * v.x - w.z * v.z, w.y * v.y - w.w * v.w,
                                    w.x * v.z + w.z * v.x, w.y * v.w + w.w * v.y);
            }
            __syncthreads();
            const float4* p4 = reinterpret_cast<const float4*>(fP) + hl * (kM3N / 4);
#pragma unroll
            for (int q = 0; q < kM3Pairs / 2; ++q) {
                const float4 a = p4[q];
                const float2 ar = make_float2(a.x, a.y), nai = make_float2(-a.z, -a.w), ai = make_float2(a.z, a.w);
#pragma unroll
                for (int j = 0; j < kM3Cpt; ++j) {
                    const float2 nr = fma2(ar, sre[j][q], mul2(nai, sim[j][q]));
                    const float2 ni = fma2(ar, sim[j][q], mul2(ai, sre[j][q]));
                    sre[j][q] = nr;
                    sim[j][q] = ni;
                }
            }
#pragma unroll kUnroll
            for (int tt = 0; tt < n; ++tt) {
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float2 xv = __bfloat1622float2(
                        *reinterpret_cast<const __nv_bfloat162*>(xs + (tt * R + r) * kM3Threads + cl));
                    const float2 x2[kM3Cpt] = {make_float2(xv.x, xv.x), make_float2(xv.y, xv.y)};
#pragma unroll
                    for (int q = 0; q < kM3N / 4; ++q) {
                        const float4 vv = fb[((tt * R + r) * kM3Heads + hl) * (kM3N / 4) + q];
#pragma unroll
                        for (int j = 0; j < kM3Cpt; ++j) {
                            sre[j][q] = fma2(make_float2(vv.x, vv.y), x2[j], sre[j][q]);
                            sim[j][q] = fma2(make_float2(vv.z, vv.w), x2[j], sim[j][q]);
                        }
                    }
                }
            }
        }

        // y of this tile's first token for this thread's channels (output r at + r xr)
        __nv_bfloat16* yp = p.y + (static_cast<int64_t>(b) * p.L + ts) * xt + c;
#pragma unroll kUnroll
        for (int tt = 0; FULL && tt < n; ++tt, yp += xt) {
            float2 xv[R];
#pragma unroll
            for (int r = 0; r < R; ++r)
                xv[r] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(xs + (tt * R + r) * kM3Threads + cl));
            // q = a q + sum_r (omega b_r) x_r, two pairs per packed register
            float2 vre[kM3Cpt][kM3Pairs / 2], vim[kM3Cpt][kM3Pairs / 2];
#pragma unroll
            for (int j = 0; j < kM3Cpt; ++j)
#pragma unroll
                for (int q = 0; q < kM3Pairs / 2; ++q) vre[j][q] = vim[j][q] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float2 x2[kM3Cpt] = {make_float2(xv[r].x, xv[r].x), make_float2(xv[r].y, xv[r].y)};
#pragma unroll
                for (int q = 0; q < kM3N / 4; ++q) {
                    const float4 bb = fb[((tt * R + r) * kM3Heads + hl) * (kM3N / 4) + q];
#pragma unroll
                    for (int j = 0; j < kM3Cpt; ++j) {
                        vre[j][q] = fma2(make_float2(bb.x, bb.y), x2[j], vre[j][q]);
                        vim[j][q] = fma2(make_float2(bb.z, bb.w), x2[j], vim[j][q]);
                    }
                }
            }
            const float4* fa4 = reinterpret_cast<const float4*>(fa) + (tt * kM3Heads + hl) * (kM3N / 4);
#pragma unroll
            for (int q = 0; q < kM3Pairs / 2; ++q) {
                const float4 a = fa4[q];              // (re, re, im, im) of pairs 2q, 2q+1
                const float2 ar = make_float2(a.x, a.y), ai = make_float2(a.z, a.w), nai = make_float2(-a.z, -a.w);
#pragma unroll
                for (int j = 0; j < kM3Cpt; ++j) {
                    const float2 nr = fma2(ar, sre[j][q], fma2(nai, sim[j][q], vre[j][q]));
                    const float2 ni = fma2(ar, sim[j][q], fma2(ai, sre[j][q], vim[j][q]));
                    sre[j][q] = nr;
                    sim[j][q] = ni;
                }
            }
            if (FULL) {
                const float* kap = fk + (tt * kM3Heads + hl) * R * R;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    // sum_k Re(conj(c_k) q_k) = sum_k (c_re q_re + c_im q_im), then kappa
                    float2 acc[kM3Cpt];
#pragma unroll
                    for (int j = 0; j < kM3Cpt; ++j) acc[j] = make_float2(0.0f, 0.0f);
#pragma unroll
                    for (int q = 0; q < kM3N / 4; ++q) {
                        const float4 cc = fc[((tt * R + r) * kM3Heads + hl) * (kM3N / 4) + q];
#pragma unroll
                        for (int j = 0; j < kM3Cpt; ++j) {
                            acc[j] = fma2(make_float2(cc.x, cc.y), sre[j][q], acc[j]);
                            acc[j] = fma2(make_float2(cc.z, cc.w), sim[j][q], acc[j]);
                        }
                    }
                    float2 yv = make_float2(acc[0].x + acc[0].y, acc[1].x + acc[1].y);
#pragma unroll
                    for (int rp = 0; rp < R; ++rp) yv = fma2(make_float2(kap[r * R + rp], kap[r * R + rp]), xv[rp], yv);
                    if (p.z) {
                        // SiLU(z) = hz + hz tanh(hz), hz = z / 2
                        const float2 zv = __bfloat1622float2(
                            *reinterpret_cast<const __nv_bfloat162*>(zs + (tt * R + r) * kM3Threads + cl));
                        const float2 hz = mul2(make_float2(0.5f, 0.5f), zv);
                        yv = mul2(yv, fma2(hz, make_float2(tanh_fast(hz.x), tanh_fast(hz.y)), hz));
                    }
                    *reinterpret_cast<__nv_bfloat162*>(yp + r * xr) = __floats2bfloat162_rn(yv.x, yv.y);
                }
            }
        }
        __syncthreads();              // the buffer and the factors are free for the next tile
    }
    cp_async_wait<0>();

    if (FULL) {
        if (chunk == p.chunks - 1) {
            // past the last token the tap weight is 0: q is the state s
            float4* hp = reinterpret_cast<float4*>(p.h_last + (static_cast<int64_t>(b) * C + c) * kM3N);
#pragma unroll
            for (int j = 0; j < kM3Cpt; ++j)
#pragma unroll
                for (int q = 0; q < kM3N / 4; ++q)
                    hp[j * (kM3N / 4) + q] = make_float4(sre[j][q].x, sim[j][q].x, sre[j][q].y, sim[j][q].y);
        }
    } else {
        float4* ep = reinterpret_cast<float4*>(
            p.ws_state + ((static_cast<int64_t>(chunk) * gridDim.z + b) * C + c) * kM3N);
#pragma unroll
        for (int j = 0; j < kM3Cpt; ++j)
#pragma unroll
            for (int q = 0; q < kM3N / 4; ++q)
                ep[j * (kM3N / 4) + q] = make_float4(sre[j][q].x, sim[j][q].x, sre[j][q].y, sim[j][q].y);
        if (tid < kM3Heads * kM3Pairs) {
            // (head h0_ + tid / pairs, pair tid % pairs)
            float* pp = p.ws_prod + ((static_cast<int64_t>(chunk) * gridDim.z + b) * p.H + h0_ + tid / kM3Pairs) * kM3N +
                        2 * (tid % kM3Pairs);
            pp[0] = prod.x;
            pp[1] = prod.y;
        }
    }
}


// ---------------------------------------------------------------- one-token step (decode)
// One token of the recurrence above per channel, in place on the state s
// (not the pre-state: the state a prefill leaves as h_last):
//     s[k] <- a[k] (s[k] + (1 - lambda) Delta u_prev[k]) + lambda Delta u[k]
//     y[r] = (sum_k Re(conj(C[r,k]) s[k]) + D x[r]) SiLU(z[r])
// with u_prev the previous token's input (x_prev, B_prev; zero when absent).
// Each channel's 16 state floats are read and written once: the step is
// bound by that HBM traffic.  A CTA covers two heads (128 channels, one per
// thread), a warp 32 channels of one head: each lane computes a[k] for pair
// k = lane mod 8 and the warp passes them round by shuffles, so no warp waits
// on another; the head's B and C rows are read by every lane of the warp
// (the same 16-byte pieces, served by L1).  The warp's 2 KB of state moves
// through shared memory so that global loads and stores are whole lines.
struct M3DecodeParams {
    const __nv_bfloat16* x;        // [B][R][H*P]
    const __nv_bfloat16* z;        // [B][R][H*P] or null
    const __nv_bfloat16* dt;       // [B][H]
    const __nv_bfloat16* trap;     // [B][H] or null (1/2)
    const float* dt_bias;          // [H] or null
    const float* A;                // [H]
    const float* theta;            // [H][N/2]
    const __nv_bfloat16* Bm;       // [B][R][G][N]
    const __nv_bfloat16* Cm;       // [B][R][G][N]
    const float* Dskip;            // [H] or null
    float* state;                  // [B][H][P][N], updated in place
    const __nv_bfloat16* x_prev;   // [B][R][H*P] or null
    const __nv_bfloat16* B_prev;   // [B][R][G][N] or null
    __nv_bfloat16* y;              // [B][R][H*P]
    int H, G;
};
constexpr int kM3DecThreads = kM3Threads;    // one channel per thread, two heads per CTA

// Position, in a warp's [32 channels][4 pieces] staging area, of 16-byte
// piece i = 4 channel + piece: XORing bits 0..1 with bits 3..4 keeps
// both the coalesced order (i = 32 q + lane) and the per-channel order
// (i = 4 lane + piece) free of shared-memory bank conflicts.
__device__ __forceinline__ int m3_dec_slot(int i) { return i ^ ((i >> 3) & 3); }

template <int R>
__global__ void __launch_bounds__(kM3DecThreads)
m3_state_update_kernel(const M3DecodeParams p)
{
    __shared__ float4 stage[kM3DecThreads / 32][32 * (kM3N / 4)];   // per warp: 32 channels' states
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, b = blockIdx.y;
    const int h = blockIdx.x * kM3Heads + tid / kM3P;      // a warp's 32 channels share one head
    const int64_t C = static_cast<int64_t>(p.H) * kM3P;
    const int64_t c = static_cast<int64_t>(blockIdx.x) * kM3Threads + tid;
    const int64_t br = static_cast<int64_t>(p.G) * kM3N;
    const int g = h * p.G / p.H;
    const bool prev = p.x_prev && p.B_prev;
    float4* st = stage[warp];

    // every load first.  The warp's 32 channel states are 2 KB of contiguous
    // memory: loaded as four 512-byte warp-wide pieces and passed through
    // shared memory, so each load and store instruction moves whole lines.
    float4* wp = reinterpret_cast<float4*>(p.state) + (static_cast<int64_t>(b) * C + (c - lane)) * (kM3N / 4);
    float4 lv[kM3N / 4];
#pragma unroll
    for (int q = 0; q < kM3N / 4; ++q) lv[q] = wp[32 * q + lane];
    const int64_t e = static_cast<int64_t>(b) * p.H + h;
    const float v = __bfloat162float(p.dt[e]) + (p.dt_bias ? p.dt_bias[h] : 0.0f);
    const float lam = p.trap ? __bfloat162float(p.trap[e]) : 0.5f;
    const float th = p.theta[h * kM3Pairs + (lane & (kM3Pairs - 1))];
    const float Ah = p.A[h];
    const float dh = p.Dskip ? p.Dskip[h] : 0.0f;
    uint4 bp[R][2], bt[R][2], ct[R][2];
    float xv[R], xp[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t ro = (static_cast<int64_t>(b) * R + r) * br + g * kM3N;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            bt[r][half] = *reinterpret_cast<const uint4*>(p.Bm + ro + 8 * half);
            ct[r][half] = *reinterpret_cast<const uint4*>(p.Cm + ro + 8 * half);
            bp[r][half] = prev ? *reinterpret_cast<const uint4*>(p.B_prev + ro + 8 * half) : make_uint4(0u, 0u, 0u, 0u);
        }
        const int64_t xi = (static_cast<int64_t>(b) * R + r) * C + c;
        xv[r] = __bfloat162float(p.x[xi]);
        xp[r] = prev ? __bfloat162float(p.x_prev[xi]) : 0.0f;
    }
#pragma unroll
    for (int q = 0; q < kM3N / 4; ++q) st[m3_dec_slot(32 * q + lane)] = lv[q];
    __syncwarp();
    float4 sv[kM3N / 4];
#pragma unroll
    for (int q = 0; q < kM3N / 4; ++q) sv[q] = st[m3_dec_slot(4 * lane + q)];   // (re, im) of pairs 2q, 2q+1

    // the head's step and tap weights (every lane), and a[k] for pair
    // k = lane mod 8, passed round the warp
    const float dl = fmaxf(v, 0.0f) + log1pf(expf(-fabsf(v)));
    const float2 w = make_float2((1.0f - lam) * dl, lam * dl);
    float sn, cs;
    m3_sincos(dl * th, &sn, &cs);
    const float mag = ex2_fast(dl * Ah * kLog2e);
    const float ar_mine = mag * cs, ai_mine = mag * sn;

    // u_prev and u: sum_r (B[r,2k] + i B[r,2k+1]) x[r]
    float2 up[kM3Pairs], u[kM3Pairs];
#pragma unroll
    for (int k = 0; k < kM3Pairs; ++k) up[k] = u[k] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint32_t bpw[4] = {bp[r][half].x, bp[r][half].y, bp[r][half].z, bp[r][half].w};
            const uint32_t btw[4] = {bt[r][half].x, bt[r][half].y, bt[r][half].z, bt[r][half].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {      // pair 4 half + j: (re, im) in one 32-bit word
                const int k = 4 * half + j;
                up[k].x = fmaf(__uint_as_float(bpw[j] << 16), xp[r], up[k].x);
                up[k].y = fmaf(__uint_as_float(bpw[j] & 0xffff0000u), xp[r], up[k].y);
                u[k].x = fmaf(__uint_as_float(btw[j] << 16), xv[r], u[k].x);
                u[k].y = fmaf(__uint_as_float(btw[j] & 0xffff0000u), xv[r], u[k].y);
            }
        }
    }
    // the state's input from the previous token, the rotation-decay, then
    // this token's input
    float2 s[kM3Pairs];
#pragma unroll
    for (int q = 0; q < kM3N / 4; ++q) {
        s[2 * q] = make_float2(fmaf(w.x, up[2 * q].x, sv[q].x), fmaf(w.x, up[2 * q].y, sv[q].y));
        s[2 * q + 1] = make_float2(fmaf(w.x, up[2 * q + 1].x, sv[q].z), fmaf(w.x, up[2 * q + 1].y, sv[q].w));
    }
#pragma unroll
    for (int k = 0; k < kM3Pairs; ++k) {
        const float ar = __shfl_sync(kFull, ar_mine, k), ai = __shfl_sync(kFull, ai_mine, k);
        const float re = fmaf(ar, s[k].x, -ai * s[k].y);
        const float im = fmaf(ar, s[k].y, ai * s[k].x);
        s[k] = make_float2(fmaf(w.y, u[k].x, re), fmaf(w.y, u[k].y, im));
    }
    // back through shared memory to whole-line stores
#pragma unroll
    for (int q = 0; q < kM3N / 4; ++q)
        st[m3_dec_slot(4 * lane + q)] = make_float4(s[2 * q].x, s[2 * q].y, s[2 * q + 1].x, s[2 * q + 1].y);
    __syncwarp();
#pragma unroll
    for (int q = 0; q < kM3N / 4; ++q) wp[32 * q + lane] = st[m3_dec_slot(32 * q + lane)];

#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t xi = (static_cast<int64_t>(b) * R + r) * C + c;
        float yv = 0.0f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint32_t cw[4] = {ct[r][half].x, ct[r][half].y, ct[r][half].z, ct[r][half].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int k = 4 * half + j;
                yv = fmaf(__uint_as_float(cw[j] << 16), s[k].x, fmaf(__uint_as_float(cw[j] & 0xffff0000u), s[k].y, yv));
            }
        }
        yv = fmaf(dh, xv[r], yv);
        if (p.z) {
            const float zv = __bfloat162float(p.z[xi]);
            yv *= zv / (1.0f + expf(-zv));
        }
        p.y[xi] = __float2bfloat16_rn(yv);
    }
}

}  // namespace mm
