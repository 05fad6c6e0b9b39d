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
// lanes per SM per clock that, not HBM, is the binding limit, so the kernel is
// laid out to spend as few fp32-pipe and issue slots as possible:
//   * a thread owns two adjacent channels and keeps their 2 x 16 states in
//     registers for its whole stretch of the sequence; every state operation,
//     and the per-token conv / softplus / SiLU / gate arithmetic, is a packed
//     f32x2 instruction over the two channels, and x, z, dt, y move as 32-bit
//     bf16 pairs;
//   * when a channel's A row is A[n] = (n+1) A[0] (detected on the device, per
//     warp), the 16 decays are powers of q = exp(Delta A[0]): one ex2 and one
//     packed multiply per state instead of 16 ex2 on the 16/clk MUFU pipe;
//   * B_t/C_t, shared by every channel of a sequence, are staged once per CTA
//     and tile in shared memory, each value duplicated into a pair, so one
//     16-byte load feeds two states of both channels;
//   * in the bf16 path SiLU is h + h tanh(h) with h = v/2 (one MUFU op), and
//     the conv weights are halved once so the conv yields v/2 directly.
//
// Parallelism.  The recurrence is sequential in t per channel: a single
// 8192-channel sequence is only 4096 channel pairs, 128 warps.  Time chunks
// supply the rest, as an exact re-association of h_t = a_t h_{t-1} + b_t:
// a summary pass finds, for each of chunks 0..K-2, its end state e_c from a
// zero start and the sum of its step sizes (whose exponential is the chunk's
// total decay P_c); the full pass starts chunk c from h0 carried through
// (P_0, e_0) .. (P_{c-1}, e_{c-1}) -- the true state at the chunk boundary --
// and runs the fused forward.  The summary pass skips the readout, the gate
// and the z/C traffic, and walks its chunk backward: e_c[n] is the sum over
// tokens of s_t B_t[n] exp(A[n] R_t), R_t the steps after token t, so with
// structured A a token's weights s r^(n+1) cost 18 packed multiplies (four
// short chains) and 16 FMAs instead of the forward recurrence's 15 decay
// powers, 16 products and 16 FMAs.  The full pass is launched as a
// programmatic dependent of the summary pass: its CTAs start on SMs the
// summary leaves free, and only those of chunks 1.. wait for the summary grid
// before the carry; the inputs were complete before the summary pass began.
//
// Latency: each tile is processed in sub-tiles of SUB tokens in three phases
// so that the long per-token chains (conv -> SiLU -> softplus -> exp) of SUB
// tokens are independent and overlap: A. per-token work, B. the state update
// (the only serial dependency is one FMA per token on each state; decay
// powers by repeated squaring), C. skip, gate and store.
//
// Data movement: each CTA owns a contiguous block of up to 256 channels of
// one sequence and one time chunk, and walks it in tiles of TILE tokens.  One
// thread stages each tile with five 3-D tiled bulk tensor copies (TMA): x
// with 3 rows of left context, z, dt, and the B_t/C_t rows, into a
// STAGES-deep ring of shared-memory buffers, each completing on its own
// mbarrier.  Rows before token 0 or past the sequence are zero-filled by the
// copy engine; the left context of token 0 is then overwritten with the
// carried conv window.  The first tiles' copies are issued before the
// per-thread setup (parameters, A rows, h0, the chunk carry), so they land
// while it runs; the setup's own global accesses move each thread's 128
// contiguous bytes in 16-byte pieces, and the chunk summaries are stored
// state-major so that a warp's access to one state is one contiguous span.
// Every wait on a copy is bounded: a copy that never lands sets a fault word
// the host can read (mamba_mixer_fault_status) instead of hanging the GPU.
#pragma once

#include <type_traits>

#include "mixer_common.cuh"

#ifndef MM_SUB
#define MM_SUB 8               // tokens per sub-tile (full pass)
#endif
#ifndef MM_SUB_SUMMARY
#define MM_SUB_SUMMARY 16      // tokens per sub-tile (summary pass: fewer live arrays, more chains)
#endif
#ifndef MM_FWD_MIN_BLOCKS
#define MM_FWD_MIN_BLOCKS 2    // resident CTAs of 128 threads per SM the register budget must allow
#endif

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
    int octets;         // channel octets (8 channels, 4 threads) per CTA
    int ctas_per_seq;   // CTAs per sequence
    int64_t chunk0_len; // tokens of time chunk 0
    int64_t chunk_len;  // tokens of every later time chunk (the last one may end early)
    int n_chunks;       // time chunks K (blockIdx.y of the full pass)
    float* ws_state;    // [K-1][batch][16][D]: end state of chunk c run from zero (state-major)
    float* ws_lsum;     // [K-1][batch][D]:     sum over chunk c of the step size l
    // Per-call status, in the caller's workspace.  hdr[0] = (epoch << 8) |
    // code of a failure (kStatusCopyTimeout, kStatusNoSummary), written by any
    // CTA that fails; hdr[1] = the epoch of the last call that ran on this
    // workspace.  The call failed iff hdr[0] >> 8 == hdr[1] and its code is set.
    unsigned long long* ws_hdr;
    // [K-1][batch][D/8]: for chunk c, sequence b and each summary-pass CTA
    // (indexed by its first channel octet), the id of the call whose summary
    // pass stored that CTA's chunk summaries.  A CTA that gave up writes none.
    unsigned long long* ws_tags;
    unsigned long long call_id;       // unique per launch pair (summary + full pass)
    unsigned long long status_epoch;  // the epoch hdr[] is written with
    int sum_octets;     // channel octets per summary-pass CTA (its tag stride)
    // Optional RMSNorm of B_t and C_t over their 16 entries before the
    // recurrence: B_t[n] * b_norm_w[n] / sqrt(mean(B_t^2) + norm_eps), the same
    // for C.  NULL = that input is used as it is.
    const float* b_norm_w;
    const float* c_norm_w;
    float norm_eps;
    int batch;
    unsigned wait_limit;  // tries per wait on a bulk copy before giving up (fault)
    int64_t check_shrink; // checked build's test hook: elements taken off y's extent (0 otherwise)
};

constexpr unsigned long long kStatusCopyTimeout = 1;  // a wait on the CTA's own bulk copies gave up
constexpr unsigned long long kStatusNoSummary = 2;    // a chunk summary this CTA starts from was not written

constexpr int kHalo = 3;   // conv left context rows (d_conv - 1)

template <typename T>
struct PrefillLayout {
    // one staged tile for a CTA of `octets` channel octets, each region
    // 128-byte aligned:
    //   x [TILE+3][ch], z [TILE][ch], dt [TILE][ch], B [TILE][16], C [TILE][16]
    __host__ __device__ static constexpr int a128(int b) { return (b + 127) & ~127; }
    __host__ __device__ static constexpr int row_bytes(int octets) { return octets * 8 * static_cast<int>(sizeof(T)); }
    __host__ __device__ static constexpr int x_bytes(int tile, int octets) { return a128((tile + kHalo) * row_bytes(octets)); }
    __host__ __device__ static constexpr int zdt_bytes(int tile, int octets) { return a128(tile * row_bytes(octets)); }
    __host__ __device__ static constexpr int bc_bytes(int tile) { return a128(tile * 16 * static_cast<int>(sizeof(T))); }
    __host__ __device__ static constexpr int stage_bytes(int tile, int octets) {
        return x_bytes(tile, octets) + 2 * zdt_bytes(tile, octets) + 2 * bc_bytes(tile);
    }
    // plus the tile's B/C in fp32, each value duplicated ([token][B0 B0 .. C15
    // C15]), and one mbarrier per stage
    __host__ __device__ static int smem_bytes(int tile, int stages, int octets) {
        return stages * stage_bytes(tile, octets) + tile * 64 * 4 + stages * 8;
    }
};

// A pair of adjacent activations <-> float2.
template <typename T> struct Pair;
template <> struct Pair<float> {
    __device__ __forceinline__ static float2 load(const float* p) { return *reinterpret_cast<const float2*>(p); }
    __device__ __forceinline__ static void store(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }
};
template <> struct Pair<__nv_bfloat16> {
    __device__ __forceinline__ static float2 load(const __nv_bfloat16* p) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
    __device__ __forceinline__ static void store(__nv_bfloat16* p, float2 v) {
        *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v.x, v.y);
    }
};

// Packed forms of the math policy's per-channel functions.
template <typename M>
__device__ __forceinline__ float2 silu2(float2 v) {
    if constexpr (M::step_scale != 1.0f) {
        // fast path: SiLU(v) = h + h tanh(h), h = v/2, with the halving and the FMA packed
        const float2 h = mul2(v, f2(0.5f, 0.5f));
        return fma2(h, f2(tanh_fast(h.x), tanh_fast(h.y)), h);
    }
    return f2(M::silu(v.x), M::silu(v.y));
}

template <typename M>
__device__ __forceinline__ float2 step_pair(float2 dt, float2 bias) {
    if constexpr (M::step_scale == 1.0f) {
        return f2(M::step(dt.x, bias.x), M::step(dt.y, bias.y));
    } else {
        // MathFast::step2 on both channels, with the affine steps packed:
        // v2 = dt log2(e) + bias2, l = max(log2(1 + 2^min(v2, 126)), v2)
        const float2 v2 = fma2(dt, f2(kLog2e, kLog2e), bias);
        const float2 e = __fadd2_rn(f2(ex2_fast(fminf(v2.x, 126.0f)), ex2_fast(fminf(v2.y, 126.0f))), f2(1.f, 1.f));
        return f2(fmaxf(lg2_fast(e.x), v2.x), fmaxf(lg2_fast(e.y), v2.y));
    }
}

template <typename M>
__device__ __forceinline__ float2 decay2(float2 l, float2 a) {
    if constexpr (M::step_scale != 1.0f) {
        // MathFast::decay on both channels with the product packed: 2^(l a)
        const float2 la = mul2(l, a);
        return f2(ex2_fast(la.x), ex2_fast(la.y));
    }
    return f2(M::decay(l.x, a.x), M::decay(l.y, a.y));
}

// SUMMARY = true: the summary pass (chunk end state from zero + sum of l).
// SUMMARY = false: the full fused forward over one chunk.
// OCT > 0: the CTA width in channel octets is the compile-time constant OCT
// (p.octets == OCT), so staged-row offsets fold into the loads' immediates;
// OCT = 0: any width.
template <typename T, typename M, int TILE, int STAGES, bool SUMMARY, int OCT = 0>
__global__ void __launch_bounds__(128, MM_FWD_MIN_BLOCKS)
mixer_fwd_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tm_x,
                 const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_dt,
                 const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c)
{
    constexpr int SUB = SUMMARY ? MM_SUB_SUMMARY : MM_SUB;
    static_assert(TILE % SUB == 0, "tile");
    constexpr bool kFast = (M::step_scale != 1.0f);
    using A_ = Act<T>;
    using P_ = Pair<T>;

    extern __shared__ __align__(128) unsigned char smem[];

    const int tid = threadIdx.x;
    const int seq = blockIdx.x / p.ctas_per_seq;
    const int blk = blockIdx.x - seq * p.ctas_per_seq;
    const int chunk = blockIdx.y;
    const int octs = OCT > 0 ? OCT : p.octets;
    const int d0 = blk * octs * 8;
    const int nch = min(octs * 8, p.D - d0);
    const int cl = 2 * tid;                      // first of my two channels, within the CTA
    const bool active = cl < nch;
    const int d = d0 + (active ? cl : 0);
    const int cls = min(cl, octs * 8 - 2);   // staged column (padding threads read a real one)
    const int64_t L = p.L;
    const int D = p.D;
    const int nthreads = OCT > 0 ? (OCT * 4 + 31) / 32 * 32 : static_cast<int>(blockDim.x);
    const int64_t t_begin = chunk == 0 ? 0 : p.chunk0_len + static_cast<int64_t>(chunk - 1) * p.chunk_len;
    const int64_t t_end = min(L, chunk == 0 ? p.chunk0_len : t_begin + p.chunk_len);

    using Lay = PrefillLayout<T>;
    const int rs = octs * 8;                     // elements per staged row (the copy box width)
    const int stageB = Lay::stage_bytes(TILE, octs);
    const int offZ = Lay::x_bytes(TILE, octs);
    const int offDT = offZ + Lay::zdt_bytes(TILE, octs);
    const int offBC = offDT + Lay::zdt_bytes(TILE, octs);
    float* bcf = reinterpret_cast<float*>(smem + STAGES * stageB);   // [TILE][64]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * stageB + TILE * 64 * 4);

    const T* xz = static_cast<const T*>(p.xz);
    const int64_t seq_row0 = static_cast<int64_t>(seq) * L;
    const int64_t chan = static_cast<int64_t>(seq) * D + d;           // (sequence, first channel) row

    // Index checks of the checked build (every one is `true` in the release
    // build): the extents, in elements, of the buffers threads address directly.
    const int64_t nBD = static_cast<int64_t>(p.batch) * D;
    const int64_t nSum = static_cast<int64_t>(p.n_chunks - 1) * nBD;  // chunk summaries per state
    auto inb = [&](int64_t first, int64_t count, int64_t extent) {
        return mm_in_bounds(first, count, extent, p.ws_hdr, p.status_epoch);
    };

    // ---------------------------------------------------------- tile loader
    const int64_t ntiles = t_end > t_begin ? (t_end - t_begin + TILE - 1) / TILE : 0;
    constexpr int kBC = SUMMARY ? 1 : 2;              // the summary pass needs B but not C (nor z)
    const unsigned rowb = static_cast<unsigned>(rs * sizeof(T));
    const unsigned stage_tx = (TILE + kHalo) * rowb + TILE * rowb * (SUMMARY ? 1 : 2) +
                              kBC * TILE * 16 * static_cast<unsigned>(sizeof(T));

    // The full pass walks its chunk forward; the summary pass walks it
    // backward (its end state is accumulated from the last token down).
    auto tile_of = [&](int64_t k) -> int64_t { return SUMMARY ? ntiles - 1 - k : k; };

    // one thread: stage the k-th tile walked (tokens t_begin + tile_of(k)*TILE ..)
    // into ring slot k % STAGES
    auto issue_tile = [&](int64_t k) {
        if (k >= ntiles) return;
        const int slot = static_cast<int>(k % STAGES);
        unsigned char* st = smem + slot * stageB;
        const int tb = static_cast<int>(t_begin + tile_of(k) * TILE);
        uint64_t* bar = &bars[slot];
        mbar_arrive_expect_tx(bar, stage_tx);
        tma_load_3d(st, &tm_x, d0, tb - kHalo, seq, bar);
        tma_load_3d(st + offDT, &tm_dt, d0, tb, seq, bar);
        tma_load_3d(st + offBC, &tm_b, 0, tb, seq, bar);
        if constexpr (!SUMMARY) {
            tma_load_3d(st + offZ, &tm_z, D + d0, tb, seq, bar);
            tma_load_3d(st + offBC + Lay::bc_bytes(TILE), &tm_c, 0, tb, seq, bar);
        }
    };

    // The full pass may be launched as a programmatic dependent of this
    // summary pass: its CTAs can then be placed on free SMs, run their setup
    // and chunk 0 meanwhile, and wait only before reading the summaries.
    if constexpr (SUMMARY) launch_dependents();
    // this call is the last one to run on the workspace
    if (!SUMMARY && blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) p.ws_hdr[1] = p.status_epoch;
    // record a failure of this CTA in the call's status and the device fault word
    auto fail = [&](unsigned long long code) {
        if (tid == 0) {
            atomicOr(&g_mm_fault, 1u);
            atomicExch(p.ws_hdr, (p.status_epoch << 8) | code);
        }
    };
    // let the copies issued for walked tiles k0 .. k0+STAGES-2 land before the
    // CTA's shared memory goes away (each wait bounded)
    auto drain = [&](int64_t k0) {
        for (int64_t j = k0; j < min(ntiles, k0 + STAGES - 1); ++j)
            mbar_wait_bounded(&bars[j % STAGES], static_cast<unsigned>((j / STAGES) & 1), 1u << 20);
    };

    // ---------------------------------------------------------- pipeline prologue (the first tiles stream in during the setup)
    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
#pragma unroll 1
        for (int s = 0; s < STAGES - 1; ++s) issue_tile(s);
    }

    // ---------------------------------------------------------- per-thread setup
    float2 w2[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) w2[k] = f2(0.f, 0.f);
    float2 cb2 = f2(0.f, 0.f), bias2 = f2(0.f, 0.f), dsk2 = f2(0.f, 0.f), A02 = f2(0.f, 0.f);
    if (active && inb(static_cast<int64_t>(d) * 4, 8, static_cast<int64_t>(D) * 4) && inb(d, 2, D)) {
        const float4 wa = *reinterpret_cast<const float4*>(p.conv_w + static_cast<int64_t>(d) * 4);
        const float4 wb = *reinterpret_cast<const float4*>(p.conv_w + static_cast<int64_t>(d + 1) * 4);
        w2[0] = f2(wa.x, wb.x); w2[1] = f2(wa.y, wb.y); w2[2] = f2(wa.z, wb.z); w2[3] = f2(wa.w, wb.w);
        if (p.conv_b) cb2 = *reinterpret_cast<const float2*>(p.conv_b + d);
        bias2 = *reinterpret_cast<const float2*>(p.dt_bias + d);
        if (p.Dskip) dsk2 = *reinterpret_cast<const float2*>(p.Dskip + d);
    }
    if constexpr (kFast) {
        bias2 = mul2(bias2, f2(kLog2e, kLog2e));
        // the conv yields v/2, the argument SiLU's tanh form needs (exact: a power-of-2 scale)
#pragma unroll
        for (int k = 0; k < 4; ++k) w2[k] = mul2(w2[k], f2(0.5f, 0.5f));
        cb2 = mul2(cb2, f2(0.5f, 0.5f));
    }
    // A pairs a2[n] = (A[d][n], A[d+1][n]): my two A rows are 128 contiguous
    // bytes, read in 16-byte loads (a warp-wide scalar load here would touch
    // 32 lines per instruction)
    float2 a2[16];
    {
        float av[32];
        const bool aok = active && inb(static_cast<int64_t>(d) * 16, 32, static_cast<int64_t>(D) * 16);
#pragma unroll
        for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(av + 4 * q) =
                aok ? __ldg(reinterpret_cast<const float4*>(p.A + static_cast<int64_t>(d) * 16) + q)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int n = 0; n < 16; ++n) a2[n] = f2(av[n], av[16 + n]);
    }
    A02 = a2[0];

    // state pairs h[n] = (h_d[n], h_{d+1}[n]), at the start of this chunk
    float2 h[16];
    if constexpr (SUMMARY) {
#pragma unroll
        for (int n = 0; n < 16; ++n) h[n] = f2(0.f, 0.f);
    } else {
        if (p.h0 && active && inb(chan * 16, 32, nBD * 16)) {
            float hv[32];   // my two channels' rows of h0: 128 contiguous bytes
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<float4*>(hv + 4 * q) = reinterpret_cast<const float4*>(p.h0 + chan * 16)[q];
#pragma unroll
            for (int n = 0; n < 16; ++n) h[n] = f2(hv[n], hv[16 + n]);
        } else {
#pragma unroll
            for (int n = 0; n < 16; ++n) h[n] = f2(0.f, 0.f);
        }
        // carry h0 through the summaries of the chunks before this one:
        // h <- exp(A sum Delta) h + e, the summaries read state-major so that
        // a warp's loads of one state are contiguous
        if (chunk > 0) {
            grid_dependency_wait();   // the summaries of chunks 0..chunk-1 (no-op when launched normally)
            // every summary-pass CTA covering my channels must have stored its
            // summaries of chunks 0..chunk-1 in this call; else the carry would
            // read stale values: record the failure and write nothing
            bool ok = true;
            if (tid == 0) {
                const int span = 8 * p.sum_octets;
                const int64_t octs = D / 8;
                for (int c = 0; c < chunk; ++c)
                    for (int sb = d0 / span; sb <= (d0 + nch - 1) / span; ++sb) {
                        const int64_t ti = (static_cast<int64_t>(c) * p.batch + seq) * octs +
                                           static_cast<int64_t>(sb) * p.sum_octets;
                        ok &= inb(ti, 1, static_cast<int64_t>(p.n_chunks - 1) * p.batch * octs) &&
                              p.ws_tags[ti] == p.call_id;
                    }
            }
            if (__syncthreads_or(!ok)) {
                fail(kStatusNoSummary);
                drain(0);
                return;
            }
        }
        if (active && chunk > 0) {
            const int64_t stride = static_cast<int64_t>(p.batch) * D;
#pragma unroll 1
            for (int c = 0; c < chunk; ++c) {
                if (!inb(c * stride + chan, 2, nSum) ||
                    !inb((c * stride + static_cast<int64_t>(seq) * D) * 16 + d, 15 * static_cast<int64_t>(D) + 2, nSum * 16))
                    continue;
                const float2 ls = *reinterpret_cast<const float2*>(p.ws_lsum + c * stride + chan);
                const float* e = p.ws_state + (c * stride + static_cast<int64_t>(seq) * D) * 16 + d;
                float2 ev[16];
#pragma unroll
                for (int n = 0; n < 16; ++n) ev[n] = *reinterpret_cast<const float2*>(e + static_cast<int64_t>(n) * D);
#pragma unroll
                for (int n = 0; n < 16; ++n) h[n] = fma2(decay2<M>(ls, a2[n]), h[n], ev[n]);
            }
        }
    }

    // Structured A (A[n] = (n+1) A[0] for every state of every channel of the
    // warp): decays are powers of q = exp(Delta A[0]).
    bool structured = false;
    if constexpr (kFast) {
        bool mine = true;
        if (active) {
#pragma unroll
            for (int n = 0; n < 16; ++n)
                mine &= (a2[n].x == static_cast<float>(n + 1) * A02.x) & (a2[n].y == static_cast<float>(n + 1) * A02.y);
        }
        structured = __all_sync(kFull, mine);
    }

    T* yg = static_cast<T*>(p.y);
    float2 lsum = f2(0.f, 0.f);           // summary pass: sum of l over the tokens walked so far

    // One sub-tile of SUB tokens starting at staged row r0 (token t0).
    // a2 (general A only): the 16 A pairs of my channels.
    auto run_sub = [&](const unsigned char* st, int r0, int64_t t0, auto structured_tag, const float2* a2) {
        constexpr bool kStruct = decltype(structured_tag)::value;
        const T* xs = reinterpret_cast<const T*>(st);          // row rho = token - 3 (tile-relative)
        [[maybe_unused]] const T* zs = reinterpret_cast<const T*>(st + offZ);   // full pass only
        const T* ds = reinterpret_cast<const T*>(st + offDT);

        // ---- A: per-token work (conv, SiLU, step, Delta*u), both channels packed
        float2 xw[SUB + 3];
#pragma unroll
        for (int k = 0; k < SUB + 3; ++k) xw[k] = P_::load(xs + (r0 + k) * rs + cls);
        float2 ea[SUB], sa[SUB], ua[SUB];
#pragma unroll
        for (int m = 0; m < SUB; ++m) {
            float2 pre = cb2;
#pragma unroll
            for (int k = 0; k < 4; ++k) pre = fma2(w2[k], xw[m + k], pre);
            float2 u;
            if constexpr (kFast) u = fma2(pre, f2(tanh_fast(pre.x), tanh_fast(pre.y)), pre);   // pre = v/2
            else u = silu2<M>(pre);
            // past the sequence end the staged dt is -inf: l = 0, so s = 0 and the decay is 1
            const float2 l = step_pair<M>(P_::load(ds + (r0 + m) * rs + cls), bias2);
            const float2 s = mul2(l, u);                         // Delta*u in B' units (B' = B * step_scale)
            if constexpr (!SUMMARY && kStruct) {
                const float2 la = mul2(l, A02);
                ea[m] = f2(ex2_fast(la.x), ex2_fast(la.y));   // q
            }
            else ea[m] = l;
            sa[m] = s;
            ua[m] = u;
        }

        if constexpr (SUMMARY) {
            // ---- B (summary pass, tokens walked last to first): the chunk's end
            // state from zero is e[n] = sum_t s_t B'_t[n] exp(A[n] R_t), with
            // R_t the sum of the steps after token t.  With R carried in lsum
            // (the steps of the tokens walked so far), a token's 16 weights are
            // s r^(n+1), r = exp(A[0] R): 18 packed multiplies, no exp per state.
            float2 R[SUB];
            R[SUB - 1] = lsum;
#pragma unroll
            for (int m = SUB - 2; m >= 0; --m) R[m] = __fadd2_rn(R[m + 1], ea[m + 1]);
            lsum = __fadd2_rn(R[0], ea[0]);
#pragma unroll
            for (int m = SUB - 1; m >= 0; --m) {
                const float* row = bcf + (r0 + m) * 64;
                if constexpr (kStruct) {
                    // weights w[n] = s r^(n+1) as four interleaved chains (step r^4),
                    // so no chain is longer than six multiplies
                    const float2 ra = mul2(R[m], A02);
                    const float2 r = f2(ex2_fast(ra.x), ex2_fast(ra.y));
                    const float2 r2 = mul2(r, r);
                    const float2 r4 = mul2(r2, r2);
                    float2 w[4];
                    w[0] = mul2(sa[m], r);
                    w[1] = mul2(w[0], r);
                    w[2] = mul2(w[0], r2);
                    w[3] = mul2(w[1], r2);
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const float4 b01 = *reinterpret_cast<const float4*>(row + 8 * g);       // (B,B) of states 4g, 4g+1
                        const float4 b23 = *reinterpret_cast<const float4*>(row + 8 * g + 4);
                        h[4 * g] = fma2(w[0], f2(b01.x, b01.y), h[4 * g]);
                        h[4 * g + 1] = fma2(w[1], f2(b01.z, b01.w), h[4 * g + 1]);
                        h[4 * g + 2] = fma2(w[2], f2(b23.x, b23.y), h[4 * g + 2]);
                        h[4 * g + 3] = fma2(w[3], f2(b23.z, b23.w), h[4 * g + 3]);
                        if (g < 3) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) w[i] = mul2(w[i], r4);
                        }
                    }
                } else {
#pragma unroll
                    for (int n = 0; n < 16; n += 2) {
                        const float4 bb = *reinterpret_cast<const float4*>(row + 2 * n);
                        h[n] = fma2(mul2(sa[m], decay2<M>(R[m], a2[n])), f2(bb.x, bb.y), h[n]);
                        h[n + 1] = fma2(mul2(sa[m], decay2<M>(R[m], a2[n + 1])), f2(bb.z, bb.w), h[n + 1]);
                    }
                }
            }
        } else {
            // ---- B: state update and readout over the SUB tokens
            float2 yacc[SUB];
#pragma unroll
            for (int m = 0; m < SUB; ++m) {
                float2 P[16];
                if constexpr (kStruct) {
                    // P[n] = q^(n+1) by repeated squaring: depth 4, 15 packed multiplies
                    P[0] = ea[m];
                    P[1] = mul2(P[0], P[0]);
                    P[2] = mul2(P[1], P[0]);
                    P[3] = mul2(P[1], P[1]);
#pragma unroll
                    for (int n = 0; n < 4; ++n) P[4 + n] = mul2(P[n], P[3]);
#pragma unroll
                    for (int n = 0; n < 8; ++n) P[8 + n] = mul2(P[n], P[7]);
                } else {
#pragma unroll
                    for (int n = 0; n < 16; ++n) P[n] = decay2<M>(ea[m], a2[n]);
                }
                const float* row = bcf + (r0 + m) * 64;
                const float2 s = sa[m];
                float2 acc0 = f2(0.f, 0.f), acc1 = f2(0.f, 0.f);
#pragma unroll
                for (int n = 0; n < 16; n += 2) {
                    const float4 bb = *reinterpret_cast<const float4*>(row + 2 * n);        // (Bn, Bn, Bn+1, Bn+1)
                    h[n] = fma2(P[n], h[n], mul2(s, f2(bb.x, bb.y)));
                    h[n + 1] = fma2(P[n + 1], h[n + 1], mul2(s, f2(bb.z, bb.w)));
                    const float4 cc = *reinterpret_cast<const float4*>(row + 32 + 2 * n);   // (Cn, Cn, Cn+1, Cn+1)
                    acc0 = fma2(f2(cc.x, cc.y), h[n], acc0);
                    acc1 = fma2(f2(cc.z, cc.w), h[n + 1], acc1);
                }
                yacc[m] = __fadd2_rn(acc0, acc1);
            }

            // ---- C: skip, gate, store (the tokens of the chunk here; every one but
            // in the sequence's last sub-tile)
#pragma unroll
            for (int m = 0; m < SUB; ++m) {
                const float2 g = silu2<M>(P_::load(zs + (r0 + m) * rs + cls));
                yacc[m] = mul2(fma2(dsk2, ua[m], yacc[m]), g);
            }
            T* yrow = yg + (seq_row0 + t0) * D + d;
            const int64_t yi = (seq_row0 + t0) * D + d;     // y's index of yrow
            if (t0 + SUB <= t_end) {
                if (active) {
#pragma unroll
                    for (int m = 0; m < SUB; ++m)
                        if (inb(yi + static_cast<int64_t>(m) * D, 2, nBD * L - p.check_shrink))
                            P_::store(yrow + m * D, yacc[m]);
                }
            } else {
                const int nvalid = static_cast<int>(t_end - t0);
#pragma unroll
                for (int m = 0; m < SUB; ++m)
                    if (m < nvalid && active && inb(yi + static_cast<int64_t>(m) * D, 2, nBD * L - p.check_shrink))
                        P_::store(yrow + m * D, yacc[m]);
            }
        }
    };

    // ---------------------------------------------------------- main loop
    const T* csi = (p.cs_in && active && inb(chan * 3, 6, nBD * 3)) ? static_cast<const T*>(p.cs_in) + chan * 3 : nullptr;
    // returns false when a copy did not land (fault set; the caller exits)
    auto main_loop = [&](auto structured_tag, const float2* a2) -> bool {
#pragma unroll 1
        for (int64_t k = 0; k < ntiles; ++k) {
            const int slot = static_cast<int>(k % STAGES);
            const bool landed = mbar_wait_bounded(&bars[slot], static_cast<unsigned>((k / STAGES) & 1), p.wait_limit);
            if (__syncthreads_or(!landed)) {
                fail(kStatusCopyTimeout);
                drain(k);
                return false;
            }
            unsigned char* st = smem + slot * stageB;
            const int64_t tile_t0 = t_begin + tile_of(k) * TILE;
            if (!SUMMARY && tile_t0 + TILE > L && cl < octs * 8) {
                // the sequence's last tile: dt = -inf past its end makes the step
                // l = softplus(-inf) = 0 there (no input, decay 1), so the sub-tile
                // code needs no per-token mask
                T* dsw = reinterpret_cast<T*>(st + offDT);
                for (int r = static_cast<int>(L - tile_t0); r < TILE; ++r) {
                    dsw[r * rs + cl] = A_::from_f32(-INFINITY);
                    dsw[r * rs + cl + 1] = A_::from_f32(-INFINITY);
                }
            }
            if (t_begin == 0 && tile_of(k) == 0 && cl < octs * 8) {
                // left context of token 0: the carried conv window (zeros if none)
                T* xs = reinterpret_cast<T*>(st);
#pragma unroll
                for (int q = 0; q < kHalo; ++q) {
                    xs[q * rs + cl] = csi ? csi[q] : A_::from_f32(0.f);
                    xs[q * rs + cl + 1] = csi ? csi[3 + q] : A_::from_f32(0.f);
                }
            }
            // B (and C) of this tile -> fp32, each value duplicated, B scaled
            {
                const T* bs = reinterpret_cast<const T*>(st + offBC);
                constexpr int cstride = Lay::bc_bytes(TILE) / static_cast<int>(sizeof(T));   // elements from B to C
                const bool normed = p.b_norm_w != nullptr || p.c_norm_w != nullptr;
                // A thread converts a pair of adjacent entries per pass (both of B or
                // both of C).  The loop's trip count and thread count are multiples of
                // 32, so each group of 8 lanes holds one 16-entry row (one token's B or
                // C) in every pass: the RMSNorm's sum of squares is three shuffles
                // within it.
                for (int i = tid; i < TILE * 8 * kBC; i += nthreads) {
                    const int r = i / (8 * kBC);
                    const int e = 2 * (i - r * 8 * kBC);          // 0..15 B, 16..31 C; even
                    const float2 v2 = P_::load(bs + (e >> 4) * cstride + r * 16 + (e & 15));
                    float va = v2.x, vb = v2.y;
                    if (normed) {
                        float ss = fmaf(va, va, vb * vb);
#pragma unroll
                        for (int o = 1; o < 8; o <<= 1) ss += __shfl_xor_sync(kFull, ss, o);
                        const float* w = (e >> 4) ? p.c_norm_w : p.b_norm_w;
                        if (w) {
                            const float sc = rsqrtf(fmaf(ss, 1.0f / 16.0f, p.norm_eps));
                            va *= sc * __ldg(w + (e & 15));
                            vb *= sc * __ldg(w + (e & 15) + 1);
                        }
                    }
                    if (e < 16) {
                        va *= M::step_scale;
                        vb *= M::step_scale;
                    }
                    *reinterpret_cast<float4*>(bcf + r * 64 + 2 * e) = make_float4(va, va, vb, vb);
                }
            }
            if (tid == 0) {
                // the slot refilled next held tile k-1, which every thread has finished with
                fence_proxy_async_smem();
                issue_tile(k + STAGES - 1);
            }
            __syncthreads();
#pragma unroll 1
            for (int j = 0; j < TILE / SUB; ++j) {
                const int r0 = (SUMMARY ? TILE / SUB - 1 - j : j) * SUB;
                run_sub(st, r0, tile_t0 + r0, structured_tag, a2);
            }
        }
        return true;
    };
    bool completed;
    if (structured) {
        completed = main_loop(std::true_type{}, nullptr);
    } else {
        completed = main_loop(std::false_type{}, a2);
    }
    if (!completed) return;

    // ---------------------------------------------------------- carried state out
    if constexpr (SUMMARY) {
        const int64_t stride = static_cast<int64_t>(p.batch) * D;
        if (active && inb(chunk * stride + chan, 2, nSum) &&
            inb((chunk * stride + static_cast<int64_t>(seq) * D) * 16 + d, 15 * static_cast<int64_t>(D) + 2, nSum * 16)) {
            float* e = p.ws_state + (chunk * stride + static_cast<int64_t>(seq) * D) * 16 + d;
#pragma unroll
            for (int n = 0; n < 16; ++n) *reinterpret_cast<float2*>(e + static_cast<int64_t>(n) * D) = h[n];
            *reinterpret_cast<float2*>(p.ws_lsum + chunk * stride + chan) = lsum;
        }
        // this CTA's summaries are stored (the full pass reads them only after
        // this grid has completed, so no fence is needed)
        __syncthreads();
        const int64_t ti = (static_cast<int64_t>(chunk) * p.batch + seq) * (D / 8) + d0 / 8;
        if (tid == 0 && inb(ti, 1, static_cast<int64_t>(p.n_chunks - 1) * p.batch * (D / 8))) p.ws_tags[ti] = p.call_id;
    } else if (active && chunk == p.n_chunks - 1 && inb(chan * 16, 32, nBD * 16) && inb(chan * 3, 6, nBD * 3)) {
        // my two channels' rows of h_last: 128 contiguous bytes, in 16-byte stores
        float4* hl = reinterpret_cast<float4*>(p.h_last + chan * 16);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            hl[q] = make_float4(h[4 * q].x, h[4 * q + 1].x, h[4 * q + 2].x, h[4 * q + 3].x);
            hl[4 + q] = make_float4(h[4 * q].y, h[4 * q + 1].y, h[4 * q + 2].y, h[4 * q + 3].y);
        }
        // the last 3 raw x of both channels, shifted in from the incoming window when L < 3
        T* cso = static_cast<T*>(p.cs_out) + chan * 3;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                const int64_t tpos = L - 3 + q;
                T v;
                if (tpos >= 0) v = inb((seq_row0 + tpos) * 2 * D + d + c, 1, nBD * L * 2) ? xz[(seq_row0 + tpos) * 2 * D + d + c]
                                                                                         : A_::from_f32(0.f);
                else v = csi ? csi[3 * c + tpos + 3] : A_::from_f32(0.f);
                cso[3 * c + q] = v;
            }
        }
    }
}

}  // namespace mm
