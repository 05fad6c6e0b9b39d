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
//   * the state lives in registers for the whole sequence (no chunk re-scan,
//     no carried partial products, nothing re-read from HBM);
//   * state pairs use packed f32x2 FMA/MUL (one issue slot per two lanes);
//   * when a channel's A row is A[n] = (n+1) A[0] (detected on the device, per
//     warp), the 16 decays are powers of q = exp(Delta A[0]): one ex2 plus one
//     packed multiply per state pair, instead of 16 ex2 on the 16/clk MUFU;
//   * the per-token work shared by a channel's states (conv, softplus, SiLU,
//     gate) runs once per (token, channel), on the lane that owns that token.
// Parallelism: the sequence is sequential per channel, so the (batch x
// d_inner) channels are the only independent units.  When they are too few
// to fill 148 SMs (a single 8192-channel sequence gives 256 warps), a
// channel's 16 states are split over LPC = 2 or 4 lanes; the lanes take turns
// computing the per-token work and exchange (decay base, Delta*u) and the
// partial readouts with warp shuffles.
//
// Data movement: each CTA owns a contiguous block of channels of one sequence
// and walks the sequence in tiles of TILE tokens.  x, z, dt rows of the block
// and the B_t/C_t rows are staged in shared memory by cp.async 16-byte copies
// in a STAGES-deep ring (rows past the sequence end are zero-filled); B/C are
// converted once per tile to fp32, permuted so each lane's states are
// contiguous, and shared by every channel of the CTA.  y is stored straight
// from the lane that owns the token.
#pragma once

#include <type_traits>

#include "mixer_common.cuh"

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
};

template <typename T>
struct PrefillLayout {
    // bytes of one staged tile for a CTA of `octets` channel octets
    __host__ __device__ static constexpr int row_bytes(int octets) { return octets * 8 * static_cast<int>(sizeof(T)); }
    __host__ __device__ static constexpr int bc_row_bytes() { return 16 * static_cast<int>(sizeof(T)); }
    __host__ __device__ static int stage_bytes(int tile, int octets) {
        return tile * (3 * row_bytes(octets) + 2 * bc_row_bytes());
    }
    __host__ __device__ static int smem_bytes(int tile, int stages, int octets) {
        return stages * stage_bytes(tile, octets) + tile * 32 * 4;
    }
};

template <typename T, typename M, int LPC, int TILE, int STAGES>
__global__ void __launch_bounds__(256)
mixer_fwd_kernel(const PrefillParams p)
{
    static_assert(LPC == 1 || LPC == 2 || LPC == 4, "lanes per channel");
    static_assert(TILE % LPC == 0, "tile");
    constexpr int NS = 16 / LPC;      // states per lane
    constexpr int NP = NS / 2;        // packed state pairs per lane
    constexpr bool kFast = (M::step_scale != 1.0f);
    using A_ = Act<T>;

    extern __shared__ __align__(16) unsigned char smem[];

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int j = tid % LPC;                  // lane within the channel
    const int cl = tid / LPC;                 // channel within the CTA
    const int seq = blockIdx.x / p.ctas_per_seq;
    const int blk = blockIdx.x - seq * p.ctas_per_seq;
    const int d0 = blk * p.octets * 8;
    const int nch = min(p.octets * 8, p.D - d0);
    const bool active = cl < nch;
    const int d = d0 + (active ? cl : 0);
    const int cls = min(cl, p.octets * 8 - 1);   // staged column (padding lanes read a real one)
    const int64_t L = p.L;
    const int D = p.D;

    const int rowB = PrefillLayout<T>::row_bytes(p.octets);
    const int stageB = PrefillLayout<T>::stage_bytes(TILE, p.octets);
    float* bcf = reinterpret_cast<float*>(smem + STAGES * stageB);   // [TILE][2][LPC][NS]

    const T* xz = static_cast<const T*>(p.xz);
    const T* dtg = static_cast<const T*>(p.dt);
    const T* Bg = static_cast<const T*>(p.Bm);
    const T* Cg = static_cast<const T*>(p.Cm);

    // ---------------------------------------------------------- tile loader
    constexpr int kElemPerChunk = 16 / sizeof(T);
    const int cpr = rowB / 16;                        // chunks per x/z/dt row
    constexpr int bcr = 16 * sizeof(T) / 16;          // chunks per B or C row
    const int chunks_per_row = 3 * cpr + 2 * bcr;
    const int nthreads = blockDim.x;
    const int64_t ntiles = (L + TILE - 1) / TILE;

    auto load_tile = [&](int64_t k) {
        if (k < ntiles) {
            unsigned char* st = smem + (k % STAGES) * stageB;
            const int total = TILE * chunks_per_row;
            for (int i = tid; i < total; i += nthreads) {
                const int r = i / chunks_per_row;
                const int c = i - r * chunks_per_row;
                const int64_t t = k * TILE + r;
                const bool tok_ok = t < L;
                const int64_t row = static_cast<int64_t>(seq) * L + (tok_ok ? t : 0);
                const void* src;
                void* dst;
                bool ok = tok_ok;
                if (c < 3 * cpr) {
                    const int which = c / cpr;             // 0: x, 1: z, 2: dt
                    const int cc = c - which * cpr;
                    ok = ok && (cc * kElemPerChunk < nch);
                    if (which == 2) src = dtg + row * D + d0 + cc * kElemPerChunk;
                    else src = xz + row * 2 * D + (which == 1 ? D : 0) + d0 + cc * kElemPerChunk;
                    dst = st + which * TILE * rowB + r * rowB + cc * 16;
                } else {
                    const int cc = c - 3 * cpr;            // [0, 2*bcr)
                    const int which = cc / bcr;            // 0: B, 1: C
                    const int part = cc - which * bcr;
                    src = (which ? Cg : Bg) + row * 16 + part * kElemPerChunk;
                    dst = st + 3 * TILE * rowB + which * TILE * 16 * sizeof(T) + r * 16 * sizeof(T) + part * 16;
                }
                cp_async16(dst, ok ? src : p.xz, ok ? 16u : 0u);
            }
        }
        cp_async_commit();
    };

    // ---------------------------------------------------------- per-lane setup
    float wsh[LPC + 3];             // conv taps shifted to this lane's token
    float cb = 0.f, bias = 0.f, dsk = 0.f;
    float a_row[NS];                // A[d, j + LPC*i]
    float A0 = 0.f;
    float h[NS];
    float xprev[3];
    {
        float w[4] = {0.f, 0.f, 0.f, 0.f};
        if (active) {
            const float4 wv = *reinterpret_cast<const float4*>(p.conv_w + static_cast<int64_t>(d) * 4);
            w[0] = wv.x; w[1] = wv.y; w[2] = wv.z; w[3] = wv.w;
            cb = p.conv_b ? p.conv_b[d] : 0.f;
            bias = p.dt_bias[d];
            dsk = p.Dskip ? p.Dskip[d] : 0.f;
        }
#pragma unroll
        for (int m = 0; m < LPC + 3; ++m) {
            float v = 0.f;
#pragma unroll
            for (int k = 0; k < 4; ++k) v = (m - j == k) ? w[k] : v;
            wsh[m] = v;
        }
        if constexpr (kFast) bias *= kLog2e;
        const float* arow = p.A + static_cast<int64_t>(d) * 16;
        A0 = active ? arow[0] : 0.f;
#pragma unroll
        for (int i = 0; i < NS; ++i) a_row[i] = active ? arow[j + LPC * i] : 0.f;
        const float* h0 = p.h0 ? p.h0 + (static_cast<int64_t>(seq) * D + d) * 16 : nullptr;
#pragma unroll
        for (int i = 0; i < NS; ++i) h[i] = (active && h0) ? h0[j + LPC * i] : 0.f;
        const T* csi = p.cs_in ? static_cast<const T*>(p.cs_in) + (static_cast<int64_t>(seq) * D + d) * 3 : nullptr;
#pragma unroll
        for (int k = 0; k < 3; ++k) xprev[k] = (active && csi) ? A_::load(csi + k) : 0.f;
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

    // One token group (LPC consecutive tokens, token r0 + j owned by this lane).
    auto run_group = [&](const unsigned char* st, const float* bct, int r0, int64_t t0, auto structured_tag) {
        constexpr bool kStruct = decltype(structured_tag)::value;
        const T* xs = reinterpret_cast<const T*>(st);
        const T* zs = reinterpret_cast<const T*>(st + TILE * rowB);
        const T* ds = reinterpret_cast<const T*>(st + 2 * TILE * rowB);
        const int rs = rowB / static_cast<int>(sizeof(T));   // elements per staged row

        // ---- per-token work of my token: conv, SiLU, step, Delta*u
        float hist[LPC + 3];
        hist[0] = xprev[0]; hist[1] = xprev[1]; hist[2] = xprev[2];
#pragma unroll
        for (int m = 0; m < LPC; ++m) hist[3 + m] = A_::to_f32(xs[(r0 + m) * rs + cls]);
        xprev[0] = hist[LPC]; xprev[1] = hist[LPC + 1]; xprev[2] = hist[LPC + 2];
        float pre = cb;
#pragma unroll
        for (int m = 0; m < LPC + 3; ++m) pre = fmaf(wsh[m], hist[m], pre);
        const float u = M::silu(pre);
        const float dtv = A_::to_f32(ds[(r0 + j) * rs + cls]);
        const float zv = A_::to_f32(zs[(r0 + j) * rs + cls]);
        const bool valid = (t0 + j) < L;
        float l;
        if constexpr (kFast) l = M::step2(dtv, bias);
        else l = M::step(dtv, bias);
        float s = l * u;            // Delta*u in B' units (B' = B * step_scale)
        if (!valid) { l = 0.f; s = 0.f; }
        float e;                    // what the lanes share: q (structured) or l
        if constexpr (kStruct) e = ex2_fast(l * A0);
        else e = l;

        // ---- the LPC tokens: decays, state update, partial readout
        float yp[LPC];
#pragma unroll
        for (int m = 0; m < LPC; ++m) {
            const float em = (LPC == 1) ? e : __shfl_sync(kFull, e, lane_base + m);
            const float sm = (LPC == 1) ? s : __shfl_sync(kFull, s, lane_base + m);
            float2 P[NP];
            if constexpr (kStruct) {
                // decays q^(n+1) for n = j + LPC*i: base q^(j+1), stride Q = q^LPC
                const float q1 = em;
                const float q2 = q1 * q1;
                float b, Q;
                if constexpr (LPC == 1) { b = q1; Q = q1; }
                else if constexpr (LPC == 2) { b = j ? q2 : q1; Q = q2; }
                else {
                    const float q3 = q2 * q1, q4 = q2 * q2;
                    b = (j & 2) ? ((j & 1) ? q4 : q3) : ((j & 1) ? q2 : q1);
                    Q = q4;
                }
                P[0] = f2(b, b * Q);
                const float QQ = Q * Q;
                const float2 step = f2(QQ, QQ);
#pragma unroll
                for (int k = 1; k < NP; ++k) P[k] = mul2(P[k - 1], step);
            } else {
#pragma unroll
                for (int k = 0; k < NP; ++k)
                    P[k] = f2(M::decay(em, a_row[2 * k]), M::decay(em, a_row[2 * k + 1]));
            }
            const float* bp = bct + ((r0 + m) * 2 + 0) * 16 + j * NS;
            const float* cp = bct + ((r0 + m) * 2 + 1) * 16 + j * NS;
            const float2 ss = f2(sm, sm);
            float2 acc = f2(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                const float2 bb = *reinterpret_cast<const float2*>(bp + 2 * k);
                const float2 cc = *reinterpret_cast<const float2*>(cp + 2 * k);
                float2 hh = f2(h[2 * k], h[2 * k + 1]);
                hh = fma2(P[k], hh, mul2(ss, bb));
                h[2 * k] = hh.x; h[2 * k + 1] = hh.y;
                acc = fma2(cc, hh, acc);
            }
            yp[m] = acc.x + acc.y;
        }

        // ---- transpose-reduce the partial readouts: lane j ends with token j
#pragma unroll
        for (int bit = LPC / 2; bit >= 1; bit >>= 1) {
            const bool upper = (j & bit) != 0;
#pragma unroll
            for (int i = 0; i < bit; ++i) {
                const float send = upper ? yp[i] : yp[i + bit];
                const float keep = upper ? yp[i + bit] : yp[i];
                yp[i] = keep + __shfl_xor_sync(kFull, send, bit);
            }
        }

        // ---- skip, gate, store
        if (valid && active) {
            const float yv = fmaf(dsk, u, yp[0]) * M::silu(zv);
            yg[(static_cast<int64_t>(seq) * L + t0 + j) * D + d] = A_::from_f32(yv);
        }
    };

    // ---------------------------------------------------------- main loop
#pragma unroll 1
    for (int64_t k = 0; k < ntiles; ++k) {
        cp_async_wait<STAGES - 2>();
        __syncthreads();
        const unsigned char* st = smem + (k % STAGES) * stageB;
        // B/C of this tile -> fp32, permuted to [r][B|C][lane j][i], B scaled
        {
            const T* bs = reinterpret_cast<const T*>(st + 3 * TILE * rowB);
            for (int i = tid; i < TILE * 32; i += nthreads) {
                const int r = i >> 5;
                const int e = i & 31;
                const int which = e >> 4;
                const int n = e & 15;
                float v = A_::to_f32(bs[which * TILE * 16 + r * 16 + n]);
                if (which == 0) v *= M::step_scale;
                bcf[(r * 2 + which) * 16 + (n % LPC) * NS + n / LPC] = v;
            }
        }
        load_tile(k + STAGES - 1);
        __syncthreads();
        const int64_t tile_t0 = k * TILE;
        if (structured) {
#pragma unroll 1
            for (int r0 = 0; r0 < TILE; r0 += LPC)
                run_group(st, bcf, r0, tile_t0 + r0, std::true_type{});
        } else {
#pragma unroll 1
            for (int r0 = 0; r0 < TILE; r0 += LPC)
                run_group(st, bcf, r0, tile_t0 + r0, std::false_type{});
        }
    }
    cp_async_wait<0>();

    // ---------------------------------------------------------- carried state out
    if (active) {
        float* hl = p.h_last + (static_cast<int64_t>(seq) * D + d) * 16;
#pragma unroll
        for (int i = 0; i < NS; ++i) hl[j + LPC * i] = h[i];
        if (j == 0) {
            // the last 3 raw x, shifted in from the incoming window when L < 3
            const T* csi = p.cs_in ? static_cast<const T*>(p.cs_in) + (static_cast<int64_t>(seq) * D + d) * 3 : nullptr;
            T* cso = static_cast<T*>(p.cs_out) + (static_cast<int64_t>(seq) * D + d) * 3;
#pragma unroll
            for (int k = 0; k < 3; ++k) {
                const int64_t tpos = L - 3 + k;
                T v;
                if (tpos >= 0) v = xz[(static_cast<int64_t>(seq) * L + tpos) * 2 * D + d];
                else v = csi ? csi[tpos + 3] : A_::from_f32(0.f);
                cso[k] = v;
            }
        }
    }
}

}  // namespace mm
