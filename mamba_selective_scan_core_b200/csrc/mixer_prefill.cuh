// Selective-scan forward (prefill) of the Mamba mixer core, fused in one pass:
// conv + SiLU, softplus step, discretisation, the fp32 recurrence, readout,
// D-skip and SiLU(z) gate.
//
// What is computed (per sequence b, channel d, state n; see the public header
// for the passages it follows):
//   u_t     = SiLU(conv_b + sum_k conv_w[k] x_{t-3+k})
//   Delta_t = softplus(dt_t + dt_bias)
//   h_t[n]  = exp(Delta_t A[n]) h_{t-1}[n] + Delta_t B_t[n] u_t
//   y_t     = (sum_n C_t[n] h_t[n] + Dskip u_t) SiLU(z_t)
//
// Why this shape on B200.  Per token and channel the recurrence does, for
// each of the 16 states, a decay, a Delta*u*B product, the state FMA and the
// readout FMA -- at least 64 fp32 pipe operations against 8 bytes of HBM
// traffic (x, z, dt in, y out; B/C are shared by all channels).  At 128 fp32
// lanes per SM per clock that is the binding limit, not HBM, so the kernel is
// laid out to spend as few fp32/issue slots as possible per state element:
//   * the state lives in registers (no re-scan of a chunk from its carried
//     state, nothing re-read from HBM);
//   * state pairs use packed f32x2 FMA/MUL (one issue slot per two lanes);
//   * when a channel's A row is A[n] = (n+1) A[0] (detected on the device, per
//     warp), the 16 decays are powers of q = exp(Delta A[0]): one ex2 plus one
//     packed multiply per state pair, instead of 16 ex2 on the 16/clk MUFU;
//   * the per-token work shared by a channel's states (conv, softplus, SiLU,
//     gate) runs once per (token, channel).
//
// Parallelism.  The recurrence is sequential in t per channel, and a single
// 8192-channel sequence is only 256 warps at one lane per channel -- under 2
// per SM.  Two ways to get more, both exact re-associations of the linear
// recurrence h_t = a_t h_{t-1} + b_t:
//   * time chunks (two passes): a summary pass runs each of chunks 0..K-2
//     from a zero state and keeps only its end state e_c and the sum of its
//     step sizes (whose exponential is the chunk's total decay P_c); the full
//     pass then starts chunk c from h0 combined with (P_0, e_0) .. (P_{c-1},
//     e_{c-1}), i.e. the true state at the chunk boundary, and runs the fused
//     forward.  The summary pass skips the readout, gate and z/C traffic.
//   * state splitting: a channel's 16 states are spread over LPC = 2 or 4
//     lanes that take turns doing the per-token work and exchange (decay
//     base, Delta*u) and the partial readouts with warp shuffles.
//
// Latency: each tile of TILE tokens is processed in sub-tiles of SUB tokens
// in three phases, so that the long per-token chains (conv -> SiLU ->
// softplus -> exp) of SUB tokens are independent and overlap:
//   A. per-token work for the SUB tokens (each lane owns every LPC-th token);
//   B. the state update for the SUB tokens (the only serial dependency is
//      one FMA per token on each state; decay powers by repeated squaring,
//      readout over two accumulators);
//   C. transpose-reduce of the partial readouts over the LPC lanes, skip,
//      gate and store, again for all SUB tokens at once.
//
// Data movement: each CTA owns a contiguous block of channels of one sequence
// and one time chunk, and walks it in tiles of TILE tokens.  x (with 3 rows
// of left context), z, dt rows of the block and the B_t/C_t rows are staged
// in shared memory by cp.async 16-byte copies in a STAGES-deep ring (rows
// outside the chunk are zero-filled; the left context of token 0 comes from
// the carried conv window); B/C are converted once per tile to fp32, permuted
// so each lane's states are contiguous, and shared by every channel of the
// CTA.
#pragma once

#include <type_traits>

#include "mixer_common.cuh"

// Scheduling knobs of the forward kernel (compile-time; the defaults are the
// measured best on B200).
#ifndef MM_SUB1
#define MM_SUB1 8              // tokens per sub-tile at one lane per channel
#endif
#ifndef MM_SUBTILE_UNROLL
#define MM_SUBTILE_UNROLL 1    // sub-tiles unrolled together (lets phases overlap)
#endif
#ifndef MM_TOKENS_OUTER
#define MM_TOKENS_OUTER 0      // phase B loop order: 0 = state pairs outer, 1 = tokens outer
#endif
#ifndef MM_MIN_BLOCKS
#define MM_MIN_BLOCKS 1        // resident CTAs per SM the register budget must allow
#endif
#define MM_PRAGMA_(x) _Pragma(#x)
#define MM_PRAGMA(x) MM_PRAGMA_(x)

namespace mm {

struct PrefillParams {
    const void* xz;
    const float* conv_w;
    const float* conv_b;
    const void* dt;
    const float* dt_bias;
    const float* A;
    const void* Bm;
    const void* Cm;
    const float* Dskip;
    const float* h0;
    const void* cs_in;
    void* y;
    float* h_last;
    void* cs_out;
    int64_t L;          // tokens per sequence
    int D;              // d_inner
    int octets;         // channel octets (8 channels) per CTA
    int ctas_per_seq;   // CTAs per sequence
    int64_t chunk_len;  // tokens per time chunk (a multiple of the tile)
    int n_chunks;       // time chunks K (blockIdx.y of the full pass)
    float* ws_state;    // [K-1][batch][D][16]: end state of chunk c run from zero
    float* ws_lsum;     // [K-1][batch][D]:     sum over chunk c of the step size l
    int batch;
};

constexpr int kHalo = 3;   // conv left context rows (d_conv - 1)

template <typename T>
struct PrefillLayout {
    // one staged tile for a CTA of `octets` channel octets:
    //   x [TILE+3][ch], z [TILE][ch], dt [TILE][ch], B [TILE][16], C [TILE][16]
    __host__ __device__ static constexpr int row_bytes(int octets) { return octets * 8 * static_cast<int>(sizeof(T)); }
    __host__ __device__ static constexpr int bc_row_bytes() { return 16 * static_cast<int>(sizeof(T)); }
    __host__ __device__ static int stage_bytes(int tile, int octets) {
        return (3 * tile + kHalo) * row_bytes(octets) + 2 * tile * bc_row_bytes();
    }
    // plus the tile's B/C in fp32, [lane j][pair k][token r][B0 B1 C0 C1], each
    // lane class's block padded by 16 bytes so the LPC classes hit different banks
    __host__ __device__ static int smem_bytes(int tile, int stages, int octets) {
        return stages * stage_bytes(tile, octets) + tile * 32 * 4 + 4 * 16;
    }
};

// Walk the chunk indices i = tid, tid + nthreads, ... of a [rows][cols] grid
// without a division per step.
struct GridWalk {
    int r, c, dr, dc, cols;
    __device__ GridWalk(int tid, int nthreads, int cols_) : cols(cols_) {
        r = tid / cols; c = tid - r * cols;
        dr = nthreads / cols; dc = nthreads - dr * cols;
    }
    __device__ void next() {
        r += dr; c += dc;
        if (c >= cols) { c -= cols; ++r; }
    }
};

// SUMMARY = true: the summary pass (chunk end state from zero + sum of l).
// SUMMARY = false: the full fused forward over one chunk.
template <typename T, typename M, int LPC, int TILE, int STAGES, bool SUMMARY>
__global__ void __launch_bounds__(256, MM_MIN_BLOCKS)
mixer_fwd_kernel(const PrefillParams p)
{
    static_assert(LPC == 1 || LPC == 2 || LPC == 4, "lanes per channel");
    constexpr int NS = 16 / LPC;          // states per lane
    constexpr int NP = NS / 2;            // packed state pairs per lane
    constexpr int SUB = LPC == 1 ? MM_SUB1 : 16;  // tokens per sub-tile
    constexpr int OWN = SUB / LPC;        // tokens of a sub-tile this lane owns
    constexpr int XW = SUB - LPC + 4;     // x window a lane reads per sub-tile
    static_assert(TILE % SUB == 0, "tile");
    constexpr bool kFast = (M::step_scale != 1.0f);
    using A_ = Act<T>;

    extern __shared__ __align__(16) unsigned char smem[];

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int j = tid % LPC;                  // lane within the channel
    const int cl = tid / LPC;                 // channel within the CTA
    const int seq = blockIdx.x / p.ctas_per_seq;
    const int blk = blockIdx.x - seq * p.ctas_per_seq;
    const int chunk = blockIdx.y;
    const int d0 = blk * p.octets * 8;
    const int nch = min(p.octets * 8, p.D - d0);
    const bool active = cl < nch;
    const int d = d0 + (active ? cl : 0);
    const int cls = min(cl, p.octets * 8 - 1);   // staged column (padding lanes read a real one)
    const int64_t L = p.L;
    const int D = p.D;
    const int nthreads = blockDim.x;
    const int64_t t_begin = static_cast<int64_t>(chunk) * p.chunk_len;
    const int64_t t_end = min(L, t_begin + p.chunk_len);

    const int rowB = PrefillLayout<T>::row_bytes(p.octets);
    const int rs = p.octets * 8;                 // elements per staged row
    const int stageB = PrefillLayout<T>::stage_bytes(TILE, p.octets);
    const int offZ = (TILE + kHalo) * rowB;
    const int offDT = offZ + TILE * rowB;
    const int offBC = offDT + TILE * rowB;
    float* bcf = reinterpret_cast<float*>(smem + STAGES * stageB);   // [LPC][NP][TILE][4] (+pad)
    constexpr int JSTRIDE = NP * TILE * 4 + 4;                         // floats per lane class

    const T* xz = static_cast<const T*>(p.xz);
    const T* dtg = static_cast<const T*>(p.dt);
    const T* Bg = static_cast<const T*>(p.Bm);
    const T* Cg = static_cast<const T*>(p.Cm);
    const int64_t seq_row0 = static_cast<int64_t>(seq) * L;
    const int64_t chan = static_cast<int64_t>(seq) * D + d;           // (sequence, channel) row

    // ---------------------------------------------------------- tile loader
    constexpr int kEPC = 16 / sizeof(T);              // elements per 16-byte chunk
    const int cpr = rowB / 16;                        // chunks per x/z/dt row
    constexpr int bcr = 16 * sizeof(T) / 16;          // chunks per B or C row
    const int64_t ntiles = t_end > t_begin ? (t_end - t_begin + TILE - 1) / TILE : 0;
    constexpr int kZDT = SUMMARY ? 1 : 2;             // the summary pass needs dt but not z
    constexpr int kBC = SUMMARY ? 1 : 2;              // ... and B but not C

    auto load_tile = [&](int64_t k) {
        if (k < ntiles) {
            unsigned char* st = smem + (k % STAGES) * stageB;
            const int64_t tbase = t_begin + k * TILE;
            // x with 3 rows of left context: staged row rho holds token tbase - 3 + rho
            for (GridWalk g(tid, nthreads, cpr); g.r < TILE + kHalo; g.next()) {
                const int64_t t = tbase - kHalo + g.r;
                const bool ok = t >= 0 && t < t_end && g.c * kEPC < nch;
                const T* src = xz + (seq_row0 + (ok ? t : 0)) * 2 * D + d0 + g.c * kEPC;
                cp_async16(st + g.r * rowB + g.c * 16, ok ? src : p.xz, ok ? 16u : 0u);
            }
            // dt (and z for the full pass)
            for (GridWalk g(tid, nthreads, kZDT * cpr); g.r < TILE; g.next()) {
                const int64_t t = tbase + g.r;
                const bool isdt = SUMMARY || g.c >= cpr;
                const int cc = (SUMMARY || !isdt) ? g.c : g.c - cpr;
                const bool ok = t < t_end && cc * kEPC < nch;
                const int64_t row = seq_row0 + (ok ? t : 0);
                const T* src = isdt ? dtg + row * D + d0 + cc * kEPC : xz + row * 2 * D + D + d0 + cc * kEPC;
                cp_async16(st + (isdt ? offDT : offZ) + g.r * rowB + cc * 16, ok ? src : p.xz, ok ? 16u : 0u);
            }
            // B (and C for the full pass)
            for (GridWalk g(tid, nthreads, kBC * bcr); g.r < TILE; g.next()) {
                const int64_t t = tbase + g.r;
                const bool isC = g.c >= bcr;
                const int part = isC ? g.c - bcr : g.c;
                const bool ok = t < t_end;
                const T* src = (isC ? Cg : Bg) + (seq_row0 + (ok ? t : 0)) * 16 + part * kEPC;
                cp_async16(st + offBC + (isC ? TILE * 16 * sizeof(T) : 0) + g.r * 16 * sizeof(T) + part * 16,
                           ok ? src : p.xz, ok ? 16u : 0u);
            }
        }
        cp_async_commit();
    };

    // ---------------------------------------------------------- per-lane setup
    float w[4] = {0.f, 0.f, 0.f, 0.f};
    float cb = 0.f, bias = 0.f, dsk = 0.f;
    float a_row[NS];                // A[d, j + LPC*i]
    float A0 = 0.f;
    float h[NS];
    if (active) {
        const float4 wv = *reinterpret_cast<const float4*>(p.conv_w + static_cast<int64_t>(d) * 4);
        w[0] = wv.x; w[1] = wv.y; w[2] = wv.z; w[3] = wv.w;
        cb = p.conv_b ? p.conv_b[d] : 0.f;
        bias = p.dt_bias[d];
        dsk = p.Dskip ? p.Dskip[d] : 0.f;
    }
    if constexpr (kFast) bias *= kLog2e;
    {
        const float* arow = p.A + static_cast<int64_t>(d) * 16;
        A0 = active ? arow[0] : 0.f;
#pragma unroll
        for (int i = 0; i < NS; ++i) a_row[i] = active ? arow[j + LPC * i] : 0.f;
        if constexpr (SUMMARY) {
#pragma unroll
            for (int i = 0; i < NS; ++i) h[i] = 0.f;
        } else {
            // state at the chunk boundary: h0 carried through the summaries of
            // the chunks before this one, h <- exp(A * sum Delta) h + e
            const float* h0 = p.h0 ? p.h0 + chan * 16 : nullptr;
#pragma unroll
            for (int i = 0; i < NS; ++i) h[i] = (active && h0) ? h0[j + LPC * i] : 0.f;
            const int64_t stride = static_cast<int64_t>(p.batch) * D;
#pragma unroll 1
            for (int c = 0; c < chunk; ++c) {
                const float ls = active ? p.ws_lsum[c * stride + chan] : 0.f;
                const float* e = p.ws_state + (c * stride + chan) * 16;
#pragma unroll
                for (int i = 0; i < NS; ++i)
                    h[i] = fmaf(M::decay(ls, a_row[i]), h[i], active ? e[j + LPC * i] : 0.f);
            }
        }
    }

    // Structured A (A[n] = (n+1) A[0] for every state of every channel of the
    // warp): decays are powers of q = exp(Delta A[0]).
    bool structured = false;
    if constexpr (kFast) {
        bool mine = true;
#pragma unroll
        for (int i = 0; i < NS; ++i) mine = mine && (a_row[i] == static_cast<float>(j + LPC * i + 1) * A0);
        structured = __all_sync(kFull, mine || !active);
    }

    // ---------------------------------------------------------- pipeline prologue
#pragma unroll 1
    for (int s = 0; s < STAGES - 1; ++s) load_tile(s);

    T* yg = static_cast<T*>(p.y);
    const int lane_base = lane & ~(LPC - 1);
    float lsum = 0.f;                   // summary pass: sum of l over my tokens

    // One sub-tile of SUB tokens starting at staged row r0 (token t0).
    auto run_sub = [&](const unsigned char* st, int r0, int64_t t0, auto structured_tag) {
        constexpr bool kStruct = decltype(structured_tag)::value;
        const T* xs = reinterpret_cast<const T*>(st);          // row rho = token - 3 (tile-relative)
        const T* zs = reinterpret_cast<const T*>(st + offZ);
        const T* ds = reinterpret_cast<const T*>(st + offDT);

        // ---- A: per-token work of my tokens r0 + LPC*i + j
        float xw[XW];                                        // x of staged rows r0+j .. r0+j+XW-1
#pragma unroll
        for (int k = 0; k < XW; ++k) xw[k] = A_::to_f32(xs[(r0 + j + k) * rs + cls]);
        float ea[OWN], sa[OWN], ua[OWN];
#pragma unroll
        for (int i = 0; i < OWN; ++i) {
            const int r = r0 + LPC * i + j;                  // tile row of this token
            float pre = cb;
#pragma unroll
            for (int k = 0; k < 4; ++k) pre = fmaf(w[k], xw[LPC * i + k], pre);
            const float u = M::silu(pre);
            const float dtv = A_::to_f32(ds[r * rs + cls]);
            float l;
            if constexpr (kFast) l = M::step2(dtv, bias);
            else l = M::step(dtv, bias);
            float s = l * u;                                 // Delta*u in B' units (B' = B * step_scale)
            const bool valid = t0 + LPC * i + j < t_end;
            if (!valid) { l = 0.f; s = 0.f; }
            if constexpr (SUMMARY) lsum += l;
            if constexpr (kStruct) ea[i] = ex2_fast(l * A0);  // q = exp(Delta A[0])
            else ea[i] = l;
            sa[i] = s;
            ua[i] = u;
        }

        // ---- B: state update over the SUB tokens.  Pairs of states outer,
        // tokens inner: each pair is a chain of SUB dependent FMAs, and the
        // NP pairs are independent of each other.
        float em[SUB], sm[SUB];
#pragma unroll
        for (int m = 0; m < SUB; ++m) {
            const int i = m / LPC, o = m % LPC;
            em[m] = (LPC == 1) ? ea[i] : __shfl_sync(kFull, ea[i], lane_base + o);
            sm[m] = (LPC == 1) ? sa[i] : __shfl_sync(kFull, sa[i], lane_base + o);
        }
        // structured decays q^(n+1), n = j + LPC*i: per token a running pair
        // (b Q^(2k), b Q^(2k+1)) with base b = q^(j+1) and stride Q = q^LPC
        float2 pw[SUB];
        float qq[SUB];
        if constexpr (kStruct) {
#pragma unroll
            for (int m = 0; m < SUB; ++m) {
                const float q1 = em[m];
                float b, Q;
                if constexpr (LPC == 1) { b = q1; Q = q1; }
                else if constexpr (LPC == 2) { const float q2 = q1 * q1; b = j ? q2 : q1; Q = q2; }
                else {
                    const float q2 = q1 * q1, q3 = q2 * q1, q4 = q2 * q2;
                    b = (j & 2) ? ((j & 1) ? q4 : q3) : ((j & 1) ? q2 : q1);
                    Q = q4;
                }
                pw[m] = f2(b, b * Q);
                qq[m] = Q * Q;
            }
        }
#if MM_TOKENS_OUTER
        float2 yacc[SUB];
        const float* bj = bcf + j * JSTRIDE + r0 * 4;
#pragma unroll
        for (int m = 0; m < SUB; ++m) {
            float2 P[NP];
            if constexpr (kStruct) {
                P[0] = pw[m];
                float st2 = qq[m];
#pragma unroll
                for (int len = 1; len < NP; len *= 2) {
                    const float2 sv = f2(st2, st2);
#pragma unroll
                    for (int k = 0; k < len; ++k)
                        if (k + len < NP) P[k + len] = mul2(P[k], sv);
                    st2 = st2 * st2;
                }
            } else {
#pragma unroll
                for (int k = 0; k < NP; ++k)
                    P[k] = f2(M::decay(em[m], a_row[2 * k]), M::decay(em[m], a_row[2 * k + 1]));
            }
            float2 acc[2];
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                const float* slot = bj + (k * TILE + m) * 4;
                float2 hh = f2(h[2 * k], h[2 * k + 1]);
                if constexpr (SUMMARY) {
                    const float2 bb = *reinterpret_cast<const float2*>(slot);
                    hh = fma2(P[k], hh, mul2(f2(sm[m], sm[m]), bb));
                } else {
                    const float4 bc = *reinterpret_cast<const float4*>(slot);
                    hh = fma2(P[k], hh, mul2(f2(sm[m], sm[m]), f2(bc.x, bc.y)));
                    acc[k & 1] = (k < 2) ? mul2(f2(bc.z, bc.w), hh) : fma2(f2(bc.z, bc.w), hh, acc[k & 1]);
                }
                h[2 * k] = hh.x; h[2 * k + 1] = hh.y;
            }
            if constexpr (!SUMMARY) yacc[m] = __fadd2_rn(acc[0], acc[1]);
        }
#else
        float2 yacc[SUB];
        const float* bj = bcf + j * JSTRIDE + r0 * 4;
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            float2 hh = f2(h[2 * k], h[2 * k + 1]);
#pragma unroll
            for (int m = 0; m < SUB; ++m) {
                const float* slot = bj + (k * TILE + m) * 4;
                float2 P;
                if constexpr (kStruct) {
                    P = pw[m];
                    if (k + 1 < NP) pw[m] = mul2(pw[m], f2(qq[m], qq[m]));
                } else {
                    P = f2(M::decay(em[m], a_row[2 * k]), M::decay(em[m], a_row[2 * k + 1]));
                }
                if constexpr (SUMMARY) {
                    const float2 bb = *reinterpret_cast<const float2*>(slot);
                    hh = fma2(P, hh, mul2(f2(sm[m], sm[m]), bb));
                } else {
                    const float4 bc = *reinterpret_cast<const float4*>(slot);
                    hh = fma2(P, hh, mul2(f2(sm[m], sm[m]), f2(bc.x, bc.y)));
                    yacc[m] = (k == 0) ? mul2(f2(bc.z, bc.w), hh) : fma2(f2(bc.z, bc.w), hh, yacc[m]);
                }
            }
            h[2 * k] = hh.x; h[2 * k + 1] = hh.y;
        }
#endif
        float yp[SUB];
        if constexpr (!SUMMARY) {
#pragma unroll
            for (int m = 0; m < SUB; ++m) yp[m] = yacc[m].x + yacc[m].y;
        }
        if constexpr (!SUMMARY) {
            // ---- C: transpose-reduce each group of LPC tokens (lane j ends with
            // token LPC*i + j), then skip, gate, store
#pragma unroll
            for (int i = 0; i < OWN; ++i) {
                float* v = yp + LPC * i;
#pragma unroll
                for (int bit = LPC / 2; bit >= 1; bit >>= 1) {
                    const bool upper = (j & bit) != 0;
#pragma unroll
                    for (int q = 0; q < bit; ++q) {
                        const float send = upper ? v[q] : v[q + bit];
                        const float keep = upper ? v[q + bit] : v[q];
                        v[q] = keep + __shfl_xor_sync(kFull, send, bit);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < OWN; ++i) {
                const int r = r0 + LPC * i + j;
                const int64_t t = t0 + LPC * i + j;
                const float zv = A_::to_f32(zs[r * rs + cls]);
                if (t < t_end && active) {
                    const float yv = fmaf(dsk, ua[i], yp[LPC * i]) * M::silu(zv);
                    yg[(seq_row0 + t) * D + d] = A_::from_f32(yv);
                }
            }
        }
    };

    // ---------------------------------------------------------- main loop
    const T* csi = p.cs_in ? static_cast<const T*>(p.cs_in) + chan * 3 : nullptr;
#pragma unroll 1
    for (int64_t k = 0; k < ntiles; ++k) {
        cp_async_wait<STAGES - 2>();
        __syncthreads();
        unsigned char* st = smem + (k % STAGES) * stageB;
        if (t_begin == 0 && k == 0 && j == 0 && cl < p.octets * 8) {
            // left context of token 0: the carried conv window (zeros if none)
            T* xs = reinterpret_cast<T*>(st);
#pragma unroll
            for (int q = 0; q < kHalo; ++q)
                xs[q * rs + cl] = (active && csi) ? csi[q] : A_::from_f32(0.f);
        }
        // B (and C) of this tile -> fp32, permuted to [r][B|C][lane j][i], B scaled
        {
            const T* bs = reinterpret_cast<const T*>(st + offBC);
            for (int i = tid; i < TILE * 16 * kBC; i += nthreads) {
                const int r = i / (16 * kBC);
                const int e = i - r * 16 * kBC;
                const int which = e >> 4;
                const int n = e & 15;
                float v = A_::to_f32(bs[which * TILE * 16 + r * 16 + n]);
                if (which == 0) v *= M::step_scale;
                const int jj = n % LPC, ii = n / LPC;      // lane class, state within lane
                bcf[jj * JSTRIDE + ((ii >> 1) * TILE + r) * 4 + which * 2 + (ii & 1)] = v;
            }
        }
        load_tile(k + STAGES - 1);
        __syncthreads();
        const int64_t tile_t0 = t_begin + k * TILE;
        if (structured) {
MM_PRAGMA(unroll MM_SUBTILE_UNROLL)
            for (int r0 = 0; r0 < TILE; r0 += SUB)
                run_sub(st, r0, tile_t0 + r0, std::true_type{});
        } else {
MM_PRAGMA(unroll MM_SUBTILE_UNROLL)
            for (int r0 = 0; r0 < TILE; r0 += SUB)
                run_sub(st, r0, tile_t0 + r0, std::false_type{});
        }
    }
    cp_async_wait<0>();

    // ---------------------------------------------------------- carried state out
    if constexpr (SUMMARY) {
#pragma unroll
        for (int bit = LPC / 2; bit >= 1; bit >>= 1) lsum += __shfl_xor_sync(kFull, lsum, bit);
        if (active) {
            const int64_t stride = static_cast<int64_t>(p.batch) * D;
            float* e = p.ws_state + (chunk * stride + chan) * 16;
#pragma unroll
            for (int i = 0; i < NS; ++i) e[j + LPC * i] = h[i];
            if (j == 0) p.ws_lsum[chunk * stride + chan] = lsum;
        }
    } else if (active && chunk == p.n_chunks - 1) {
        float* hl = p.h_last + chan * 16;
#pragma unroll
        for (int i = 0; i < NS; ++i) hl[j + LPC * i] = h[i];
        if (j == 0) {
            // the last 3 raw x, shifted in from the incoming window when L < 3
            T* cso = static_cast<T*>(p.cs_out) + chan * 3;
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                const int64_t tpos = L - 3 + q;
                T v;
                if (tpos >= 0) v = xz[(seq_row0 + tpos) * 2 * D + d];
                else v = csi ? csi[tpos + 3] : A_::from_f32(0.f);
                cso[q] = v;
            }
        }
    }
}

}  // namespace mm
