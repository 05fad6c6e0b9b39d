// The Mamba-2 form of the selective scan on the fifth-generation tensor cores.
//
// The lesson's "SSM in one page" section: Mamba-2 simplified the state matrix
// (to a scalar times the identity, per head), and its "Mamba-3" section:
// Mamba-2 discretises with Euler's rule.  Per head h (P channels, state N x P),
// with a_t = Delta_t A[h] and Delta_t = softplus(dt_t[h] + dt_bias[h]):
//
//     h_t = exp(a_t) h_{t-1} + Delta_t x_t B_t^T        (x_t: P, B_t: N)
//     y_t = h_t C_t + D[h] x_t,   gated by SiLU(z_t)
//
// A scalar decay makes the recurrence over a chunk of Q tokens a sum of
// dense products.  With cum_i = a_{t0} + ... + a_i (the chunk's inclusive
// prefix sum) and H_in the state entering the chunk:
//
//     y_i   = sum_{j<=i} (C_i . B_j) exp(cum_i - cum_j) Delta_j x_j   (intra-chunk)
//           + exp(cum_i) C_i H_in  +  D x_i                            (carried state)
//     H_out = exp(cum_end) H_in + sum_j exp(cum_end - cum_j) Delta_j x_j B_j^T
//
// That is the same recurrence with its sums regrouped (exact up to rounding
// order).  Three kernels, Q = 128 tokens per chunk:
//
//   ssd_chunk_state_kernel (chunk, head, batch): S_c = sum_j w_j B_j x_j^T
//       with w_j = exp(cum_end - cum_j) Delta_j -- one tcgen05 product
//       [N x Q] . [Q x P] -- and the chunk's total decay exp(cum_end);
//   ssd_state_pass_kernel (state entries): H_in[c] = H (as hi and lo bf16
//       parts), H = dec_c H + S_c over the chunks in order, from h0 (fp32);
//       the last H is h_last;
//   ssd_chunk_scan_kernel (chunk, head, batch): G = C B^T (tcgen05), the
//       masked, decayed M = G o L (+ D on the diagonal) in shared memory,
//       then Y = M X + exp(cum) (C H_in^T) (tcgen05), gated and stored.
//
// Operands of every product sit in shared memory in the K-major, 128-byte
// swizzled layout; C, B and H_in arrive there by bulk tensor copies, the
// transposed x and the weighted B^T and M are written by the threads.  fp32
// accumulation in tensor memory.  x, B and C are bf16 inputs, exact as
// operands; an operand the kernels compute (w B, M, the carried state) is
// split into two bf16 parts, hi = bf16(v) and lo = bf16(v - hi), and its
// product is taken twice and summed: about 16 significant bits over the fp32
// range, where a single bf16 rounding (8 bits) would put a 2^-9 relative error
// on every term of the sums.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "mixer_common.cuh"
#include "proj_gemm.cuh"

namespace mm {

constexpr int kSsdQ = 128;        // tokens per chunk (the products' M)
constexpr int kSsdP = 64;         // channels per head
constexpr int kSsdN = 128;        // d_state
constexpr int kSsdThreads = 128;  // one token (or one state row) per thread
constexpr int kSsdScanThreads = 256;   // the chunk scan: two warpgroups share each row

struct SsdParams {
    const __nv_bfloat16* x;      // [B][L][H*P]
    const __nv_bfloat16* z;      // [B][L][H*P] or null (no gate)
    const __nv_bfloat16* dt;     // [B][L][H]
    const float* dt_bias;        // [H] or null
    const float* A;              // [H]
    const __nv_bfloat16* Bm;     // [B][L][G*N]
    const __nv_bfloat16* Cm;     // [B][L][G*N]
    const float* Dskip;          // [H] or null
    const float* h0;             // [B][H][P][N] or null
    __nv_bfloat16* y;            // [B][L][H*P]
    float* h_last;               // [B][H][P][N]
    float* S;                    // [B][chunks][H][P][N]  chunk states from zero (workspace)
    __nv_bfloat16* Hin;          // [2][B][chunks][H][P][N] state entering each chunk, hi then lo parts (workspace)
    int64_t hin_lo;              // elements from the hi parts to the lo parts
    float* dec;                  // [B][H][chunks]        exp(cum_end) of each chunk (workspace)
    int64_t L;
    int H, G, chunks, batch;
    unsigned wait_limit;
    unsigned long long* status;  // [0] (epoch << 8) | code of a failure, [1] the call's epoch; or null
    unsigned long long status_epoch;
};

// Byte offset of 16-byte piece `piece` (0..7) of row r in one K-block (rows x
// 64 bf16, 128 bytes a row) of the K-major, 128-byte-swizzled layout: rows
// 128 bytes apart, 8-row groups 1024 bytes apart, the piece index XORed with
// the row's index within its group.  The block starts on a 1024-byte boundary.
__device__ __forceinline__ uint32_t sw128_off(int r, int piece) {
    return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((piece ^ (r & 7)) << 4));
}
// element (r, k), k < 128, of a [rows][128] tile made of two such K-blocks
__device__ __forceinline__ uint32_t sw128_elem(int rows, int r, int k) {
    return static_cast<uint32_t>((k >> 6) * rows * 128) + sw128_off(r, (k & 63) >> 3) + (k & 7) * 2;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// v = hi + lo to about 16 significant bits: hi = bf16(v), lo = bf16(v - hi)
__device__ __forceinline__ void split_bf16(float v, __nv_bfloat16& hi, __nv_bfloat16& lo) {
    hi = __float2bfloat16_rn(v);
    lo = __float2bfloat16_rn(v - __bfloat162float(hi));
}
// the same for a pair, packed low element first
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
    hi = pack_bf16x2(a, b);
    lo = pack_bf16x2(a - bf16_lo(hi), b - bf16_hi(hi));
}

// One contiguous bulk copy shared -> global (16-byte aligned, a multiple of
// 16 bytes), in this thread's bulk group.
__device__ __forceinline__ void bulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;\n"
                 :: "l"(reinterpret_cast<uint64_t>(gdst)), "r"(smem_addr(ssrc)), "r"(bytes) : "memory");
}
// 3-D tiled bulk tensor copy shared -> global (a store; rows and columns
// outside the tensor are not written), in this thread's bulk group.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3}], [%4];\n"
                 :: "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(src)) : "memory");
}

__device__ __forceinline__ void ssd_fail(const SsdParams& p) {
    atomicOr(&g_mm_fault, 1u);
    if (p.status) atomicExch(p.status, (p.status_epoch << 8) | 1ull);
}

// Step size and the inclusive prefix sum of Delta A over the chunk, one token
// per thread (tokens past the sequence contribute nothing).  Leaves, per token
// j of the chunk, Delta_j in delta[j] and cum_j * log2(e) in cum2[j]; returns
// this thread's Delta.  Contains __syncthreads.
__device__ __forceinline__ void ssd_chunk_prefix(const SsdParams& p, int b, int h, int64_t t0, float* delta,
                                                 float* cum2, float* warp_sums) {
    const int j = threadIdx.x, lane = j & 31, warp = j >> 5;   // token j of the chunk (threads past Q idle)
    const int64_t t = t0 + j;
    float dl = 0.0f;
    if (j < kSsdQ && t < p.L) {
        const float v = __bfloat162float(p.dt[(static_cast<int64_t>(b) * p.L + t) * p.H + h]) +
                        (p.dt_bias ? p.dt_bias[h] : 0.0f);
        dl = fmaxf(v, 0.0f) + log1pf(expf(-fabsf(v)));
    }
    float v = dl * p.A[h] * kLog2e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float n = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31 && j < kSsdQ) warp_sums[warp] = v;
    __syncthreads();
    if (j < kSsdQ) {
        for (int w = 0; w < warp; ++w) v += warp_sums[w];
        delta[j] = dl;
        cum2[j] = v;
    }
    __syncthreads();
}

// ---------------------------------------------------------------- MN-major operands
// Shared-memory descriptor of an MN-major operand tile as a 128-byte swizzled
// tensor copy writes it: along M (or N) 64 bf16 per 128-byte row, one row per
// k, 8-row groups 1024 bytes apart (stride byte offset), 64-wide M/N blocks
// `lbo` bytes apart (leading byte offset; 0 for a single block).  Version 1,
// 128-byte swizzle; the tile starts on a 1024-byte boundary, and a K step of
// 16 advances the start by two groups (2048 bytes).
__device__ __forceinline__ uint64_t umma_desc_sw128_mn(uint32_t smem_byte_addr, uint32_t lbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_byte_addr >> 4) & 0x3FFF);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
    d |= static_cast<uint64_t>(1024 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}
// instruction descriptor of kind::f16 (bf16 operands, fp32 accumulator) with
// A and/or B MN-major (bits 15 and 16)
__host__ __device__ constexpr uint32_t umma_idesc_bf16_mn(int m, int n, bool a_mn, bool b_mn) {
    return umma_idesc_bf16(m, n) | (a_mn ? 1u << 15 : 0u) | (b_mn ? 1u << 16 : 0u);
}

// ---------------------------------------------------------------- chunk states
// S[n][p] = sum_j B_j[n] (w_j x_j[p]): A = B as copied ([token][n], MN-major,
// two 64-wide blocks of n), B = the x tile as copied ([token][p], MN-major),
// each row scaled in place by its w_j and split into hi and lo parts.
struct SsdStateLayout {
    static constexpr int b_bytes = kSsdQ * kSsdN * 2;     // B [Q rows][N]: two [Q][64] blocks   32 KB
    static constexpr int x_bytes = kSsdQ * kSsdP * 2;     // x [Q rows][P], then hi of w x      16 KB; lo 16 KB
    static constexpr int f_off = b_bytes + 2 * x_bytes;
    static constexpr int smem_bytes = 1024 + f_off + 2 * kSsdQ * 4 + 16 + 2 * 8 + 16;
    static constexpr uint32_t tx_bytes = b_bytes + x_bytes;
};

__global__ void __launch_bounds__(kSsdThreads, 3)
ssd_chunk_state_kernel(const SsdParams p, const __grid_constant__ CUtensorMap tm_b,
                       const __grid_constant__ CUtensorMap tm_x)
{
    using Lay = SsdStateLayout;
    extern __shared__ __align__(1024) unsigned char ssm_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(ssm_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* bt = sm;
    unsigned char* xh = sm + Lay::b_bytes;
    unsigned char* xl = xh + Lay::x_bytes;
    float* delta = reinterpret_cast<float*>(sm + Lay::f_off);
    float* cum2 = delta + kSsdQ;
    float* warp_sums = cum2 + kSsdQ;                      // 4 floats
    uint64_t* bars = reinterpret_cast<uint64_t*>(warp_sums + 4);   // loaded, products done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);

    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int64_t t0 = static_cast<int64_t>(c) * kSsdQ;
    const int g = h / (p.H / p.G);

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
        // B and x rows of the chunk (rows past the sequence read as zeros)
        mbar_arrive_expect_tx(&bars[0], Lay::tx_bytes);
        const int tok = static_cast<int>(t0);
        tma_load_3d(bt, &tm_b, g * kSsdN, tok, b, &bars[0]);
        tma_load_3d(bt + kSsdQ * 128, &tm_b, g * kSsdN + 64, tok, b, &bars[0]);
        tma_load_3d(xh, &tm_x, h * kSsdP, tok, b, &bars[0]);
    }
    if (warp == 2) {
        tmem_alloc(tmem_slot, 64);
        tmem_relinquish();
        tc_fence_before();
    }
    ssd_chunk_prefix(p, b, h, t0, delta, cum2, warp_sums);   // syncs: the barriers and tensor memory are set up
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const bool loaded = __syncthreads_and(mbar_wait_bounded(&bars[0], 0, p.wait_limit));
    if (loaded) {
        // row j of the x tile (its 16-byte pieces in swizzled order, which a
        // scale of the whole row does not see) times w_j = exp(cum_end - cum_j)
        // Delta_j, as hi and lo parts
        const int j = tid;
        const float w = t0 + j < p.L ? ex2_fast(cum2[kSsdQ - 1] - cum2[j]) * delta[j] : 0.0f;
        uint4* rh = reinterpret_cast<uint4*>(xh + j * 128);
        uint4* rl = reinterpret_cast<uint4*>(xl + j * 128);
#pragma unroll
        for (int q0 = 0; q0 < 8; ++q0) {
            const int q = q0 ^ (j & 7);     // lanes j..j+7 start on different banks
            const uint4 v = rh[q];
            uint4 hi, lo;
            split_bf16x2(w * bf16_lo(v.x), w * bf16_hi(v.x), hi.x, lo.x);
            split_bf16x2(w * bf16_lo(v.y), w * bf16_hi(v.y), hi.y, lo.y);
            split_bf16x2(w * bf16_lo(v.z), w * bf16_hi(v.z), hi.z, lo.z);
            split_bf16x2(w * bf16_lo(v.w), w * bf16_hi(v.w), hi.w, lo.w);
            rh[q] = hi;
            rl[q] = lo;
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // M = N = 128, N = P = 64, K = Q = 128; both operands MN-major
    if (loaded && warp == 1 && elect_one_lane()) {
        constexpr uint32_t idesc = umma_idesc_bf16_mn(kSsdN, kSsdP, true, true);
        const uint32_t a0 = smem_addr(bt), h0 = smem_addr(xh), l0 = smem_addr(xl);
#pragma unroll
        for (int kk = 0; kk < kSsdQ / 16; ++kk) {
            const uint32_t koff = kk * 2048;
            const uint64_t adesc = umma_desc_sw128_mn(a0 + koff, kSsdQ * 128);
            umma_bf16(tmem, adesc, umma_desc_sw128_mn(h0 + koff, 0), idesc, kk > 0 ? 1u : 0u);
            umma_bf16(tmem, adesc, umma_desc_sw128_mn(l0 + koff, 0), idesc, 1u);
        }
        umma_commit(&bars[1]);
    }
    bool ok = false;
    if (loaded) ok = mbar_wait_bounded(&bars[1], 0, p.wait_limit);
    tc_fence_after();
    if (__syncthreads_and(ok)) {
        // thread n owns state row n; the [P][N] block S[b][c][h], contiguous
        // in the workspace, is staged in B's tile (free now) and written out
        // by one bulk copy
        const int n = tid;
        float* stage = reinterpret_cast<float*>(bt);
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            float v[32];
            tmem_ld32(lane_base + half * 32, v);
#pragma unroll
            for (int q = 0; q < 32; ++q) stage[(half * 32 + q) * kSsdN + n] = v[q];
        }
        // the staging writes, before the bulk copy reads them
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            bulk_store(p.S + ((static_cast<int64_t>(b) * p.chunks + c) * p.H + h) * (kSsdP * kSsdN), stage,
                       kSsdP * kSsdN * 4);
            bulk_commit_group();
            p.dec[(static_cast<int64_t>(b) * p.H + h) * p.chunks + c] = ex2_fast(cum2[kSsdQ - 1]);
            // the copy has read shared memory before the CTA ends
            bulk_wait_read_all();
        }
    } else {
        if (tid == 0) ssd_fail(p);
        // the copies and products finish before shared and tensor memory go away
        if (warp == 1 && elect_one_lane()) {
            if (!loaded) mbar_wait_bounded(&bars[0], 0, 1u << 20);
            else mbar_wait_bounded(&bars[1], 0, 1u << 20);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
}

// ---------------------------------------------------------------- state passing
// One thread: 4 consecutive state entries (same head, channel; n..n+3) of one
// sequence, walked through every chunk in order.
__global__ void __launch_bounds__(256)
ssd_state_pass_kernel(const SsdParams p)
{
    constexpr int64_t kHead = int64_t(kSsdP) * kSsdN;
    constexpr int kAhead = 4;     // chunks whose S is requested before their H_in stores
    const int64_t per_seq = int64_t(p.H) * kHead;
    const int64_t f = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
    // the call's epoch for its status word (this launch always runs)
    if (p.status && f == 0 && blockIdx.y == 0) p.status[1] = p.status_epoch;
    if (f >= per_seq) return;
    const int b = blockIdx.y;
    const int h = static_cast<int>(f / kHead);
    float4 s = p.h0 ? *reinterpret_cast<const float4*>(p.h0 + b * per_seq + f) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float* dec = p.dec + (static_cast<int64_t>(b) * p.H + h) * p.chunks;
    const float* __restrict__ S = p.S;
    // Two groups of kAhead chunks' S in registers: the next group's loads are
    // issued before the current group is passed on, so the stream of loads
    // does not stop at each group's end.
    float4 addA[kAhead], addB[kAhead];
    float dA[kAhead], dB[kAhead];
    auto load = [&](float4 (&add)[kAhead], float (&d)[kAhead], int c0) {
#pragma unroll
        for (int j = 0; j < kAhead; ++j) {
            if (c0 + j < p.chunks) {
                add[j] = __ldcs(reinterpret_cast<const float4*>(S + (static_cast<int64_t>(b) * p.chunks + c0 + j) * per_seq + f));
                d[j] = dec[c0 + j];
            }
        }
    };
    auto pass = [&](const float4 (&add)[kAhead], const float (&d)[kAhead], int c0) {
#pragma unroll
        for (int j = 0; j < kAhead; ++j) {
            if (c0 + j < p.chunks) {
                const int64_t off = (static_cast<int64_t>(b) * p.chunks + c0 + j) * per_seq + f;
                uint2 hi, lo;
                split_bf16x2(s.x, s.y, hi.x, lo.x);
                split_bf16x2(s.z, s.w, hi.y, lo.y);
                *reinterpret_cast<uint2*>(p.Hin + off) = hi;
                *reinterpret_cast<uint2*>(p.Hin + p.hin_lo + off) = lo;
                s.x = fmaf(d[j], s.x, add[j].x);
                s.y = fmaf(d[j], s.y, add[j].y);
                s.z = fmaf(d[j], s.z, add[j].z);
                s.w = fmaf(d[j], s.w, add[j].w);
            }
        }
    };
    load(addA, dA, 0);
    for (int c0 = 0; c0 < p.chunks; c0 += 2 * kAhead) {
        load(addB, dB, c0 + kAhead);
        pass(addA, dA, c0);
        load(addA, dA, c0 + 2 * kAhead);
        pass(addB, dB, c0 + kAhead);
    }
    *reinterpret_cast<float4*>(p.h_last + b * per_seq + f) = s;
}

// ---------------------------------------------------------------- chunk scan
// Shared memory of the chunk scan.  The first products read C, B and H_in;
// once they complete, the same space holds M (hi over B, lo over H_in) and
// the x tile (over C, MN-major: [token][p]) for the second.
struct SsdScanLayout {
    static constexpr int c_off = 0;                                 // C [Q rows][N] 32 KB, then x [Q rows][P]
    static constexpr int b_off = c_off + kSsdQ * kSsdN * 2;         // B [Q rows][N] 32 KB, then M hi [Q rows][Q]
    static constexpr int h_off = b_off + kSsdQ * kSsdN * 2;         // H_in hi, lo [P rows][N] 2 x 16 KB, then M lo
    static constexpr int hin_bytes = kSsdP * kSsdN * 2;
    static constexpr int f_off = h_off + 2 * hin_bytes;             // delta, cum2, warp sums, column factors
    static constexpr int bar_off = f_off + 3 * kSsdQ * 4 + 16;
    static constexpr int smem_bytes = 1024 + bar_off + 4 * 8 + 16;
    static constexpr uint32_t tx_bytes = 2 * kSsdQ * kSsdN * 2 + 2 * hin_bytes;
};
static_assert(SsdScanLayout::b_off % 1024 == 0 && SsdScanLayout::h_off % 1024 == 0 &&
              SsdScanLayout::hin_bytes % 1024 == 0, "operand tiles start on 1024-byte boundaries");

// Tensor memory columns of the chunk scan: G [Q x Q], C H_in^T [Q x P], M X [Q x P].
constexpr uint32_t kSsdColG = 0, kSsdColOff = 128, kSsdColDiag = 192, kSsdCols = 256;

__global__ void __launch_bounds__(kSsdScanThreads, 2)
ssd_chunk_scan_kernel(const SsdParams p, const __grid_constant__ CUtensorMap tm_c,
                      const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_h,
                      const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_z,
                      const __grid_constant__ CUtensorMap tm_y)
{
    using Lay = SsdScanLayout;
    extern __shared__ __align__(1024) unsigned char ssc_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(ssc_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* ct = sm + Lay::c_off;      // C, then x
    unsigned char* bt = sm + Lay::b_off;      // B, then M hi
    unsigned char* ht = sm + Lay::h_off;      // H_in hi and lo, then M lo
    float* delta = reinterpret_cast<float*>(sm + Lay::f_off);
    float* cum2 = delta + kSsdQ;
    float* warp_sums = cum2 + kSsdQ;
    float* colf = warp_sums + 4;          // exp(cum_j0 - cum_j) Delta_j, j0 the first column of j's 32-column block
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::bar_off);   // loaded, products 1, product 2, x loaded
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);

    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, wg = warp >> 2;   // tensor-memory lane quarter; warpgroup
    const int64_t t0 = static_cast<int64_t>(c) * kSsdQ;
    const int g = h / (p.H / p.G);

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_init(&bars[2], 1);
        mbar_init(&bars[3], 1);
        fence_mbar_init();
        // C and B rows of the chunk (rows past the sequence read as zeros), and
        // the state entering it (hi and lo parts): two 64-wide K-blocks each
        mbar_arrive_expect_tx(&bars[0], Lay::tx_bytes);
        const int tok = static_cast<int>(t0);
        const int hrow = static_cast<int>(((static_cast<int64_t>(b) * p.chunks + c) * p.H + h) * kSsdP);
        const int lo_rows = static_cast<int>(p.hin_lo / kSsdN);
        for (int kb = 0; kb < 2; ++kb) {
            tma_load_3d(ct + kb * (kSsdQ * 128), &tm_c, g * kSsdN + kb * 64, tok, b, &bars[0]);
            tma_load_3d(bt + kb * (kSsdQ * 128), &tm_b, g * kSsdN + kb * 64, tok, b, &bars[0]);
            tma_load_3d(ht + kb * (kSsdP * 128), &tm_h, kb * 64, hrow, 0, &bars[0]);
            tma_load_3d(ht + Lay::hin_bytes + kb * (kSsdP * 128), &tm_h, kb * 64, lo_rows + hrow, 0, &bars[0]);
        }
    }
    if (warp == 2) {
        tmem_alloc(tmem_slot, kSsdCols);
        tmem_relinquish();
        tc_fence_before();
    }
    ssd_chunk_prefix(p, b, h, t0, delta, cum2, warp_sums);   // syncs
    // The decay of M's element (i, j) factors within j's 32-column block:
    // exp(cum_i - cum_j) = exp(cum_i - cum_j0) exp(cum_j0 - cum_j), the second
    // factor (with Delta_j) once per column here, the first once per row and
    // block below.  A block whose own decay range exceeds 2^60 keeps one
    // exponential per element instead (no overflow, no lost small terms).
    if (tid < kSsdQ) colf[tid] = ex2_fast(cum2[tid & ~31] - cum2[tid]) * delta[tid];
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);

    // products 1: G = C B^T (N = Q) and C H_in^T (N = P, hi and lo), K = N = 128
    bool loaded = true, ok = true;
    bool x_issued = false, x_done = false;    // the x tile's copy (warp 1's elected lane)
    if (warp == 1 && elect_one_lane()) {
        loaded = mbar_wait_bounded(&bars[0], 0, p.wait_limit);
        if (loaded) {
            tc_fence_after();
            constexpr uint32_t id_g = umma_idesc_bf16(kSsdQ, kSsdQ);
            constexpr uint32_t id_o = umma_idesc_bf16(kSsdQ, kSsdP);
            const uint32_t ca = smem_addr(ct), ba = smem_addr(bt), ha = smem_addr(ht);
#pragma unroll
            for (int kk = 0; kk < kSsdN / 16; ++kk) {
                const uint32_t koff = (kk & 3) * 32;
                const uint64_t adesc = umma_desc_sw128(ca + (kk >> 2) * (kSsdQ * 128) + koff);
                umma_bf16(tmem + kSsdColG, adesc, umma_desc_sw128(ba + (kk >> 2) * (kSsdQ * 128) + koff), id_g,
                          kk > 0 ? 1u : 0u);
                const uint32_t hk = ha + (kk >> 2) * (kSsdP * 128) + koff;
                umma_bf16(tmem + kSsdColOff, adesc, umma_desc_sw128(hk), id_o, kk > 0 ? 1u : 0u);
                umma_bf16(tmem + kSsdColOff, adesc, umma_desc_sw128(hk + Lay::hin_bytes), id_o, 1u);
            }
            umma_commit(&bars[1]);
            // C is free once these products complete: the x tile (and the
            // gate's z tile after it) go there, copied while M is built
            if (mbar_wait_bounded(&bars[1], 0, p.wait_limit)) {
                mbar_arrive_expect_tx(&bars[3], (p.z ? 2 : 1) * kSsdQ * kSsdP * 2);
                tma_load_3d(ct, &tm_x, h * kSsdP, static_cast<int>(t0), b, &bars[3]);
                if (p.z) tma_load_3d(ct + kSsdQ * kSsdP * 2, &tm_z, h * kSsdP, static_cast<int>(t0), b, &bars[3]);
                x_issued = true;
            }
        }
    }
    const bool issued1 = __syncthreads_and(loaded);
    if (issued1) ok = mbar_wait_bounded(&bars[1], 0, p.wait_limit);
    tc_fence_after();
    const bool g_ready = __syncthreads_and(issued1 && ok);

    // M[i][j] = G[i][j] exp(cum_i - cum_j) Delta_j for j <= i, 0 above the
    // diagonal, plus D on it; row i as hi and lo parts over the B and H_in
    // tiles (both free now).  Row i belongs to lane quarter i / 32; the two
    // warpgroups take its even and odd 32-column blocks.
    const int i = quarter * 32 + lane;
    if (g_ready) {
        const float ci = cum2[i];
        const float dsk = p.Dskip ? p.Dskip[h] : 0.0f;
#pragma unroll 1
        for (int jb = wg; jb < kSsdQ / 32; jb += 2) {
            float m[32];
            if (jb <= quarter) {     // warp-uniform: blocks above the diagonal block are zero
                tmem_ld32(lane_base + kSsdColG + jb * 32, m);
                const float c0 = cum2[jb * 32];
                if (c0 - cum2[jb * 32 + 31] <= 60.0f) {     // the same for every thread of the CTA
                    const float ei = ex2_fast(ci - c0);
                    const float4* cf4 = reinterpret_cast<const float4*>(colf + jb * 32);
                    if (jb < quarter) {
                        // a block below the diagonal block: every j < i
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4) {
                            const float4 cf = cf4[q4];
                            m[4 * q4] = m[4 * q4] * ei * cf.x;
                            m[4 * q4 + 1] = m[4 * q4 + 1] * ei * cf.y;
                            m[4 * q4 + 2] = m[4 * q4 + 2] * ei * cf.z;
                            m[4 * q4 + 3] = m[4 * q4 + 3] * ei * cf.w;
                        }
                    } else {
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4) {
                            const float4 cf = cf4[q4];
                            const float cv[4] = {cf.x, cf.y, cf.z, cf.w};
#pragma unroll
                            for (int e4 = 0; e4 < 4; ++e4) {
                                const int q = 4 * q4 + e4, j = jb * 32 + q;
                                m[q] = j <= i ? m[q] * ei * cv[e4] : 0.0f;
                                if (j == i) m[q] += dsk;
                            }
                        }
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q) {
                        const int j = jb * 32 + q;
                        m[q] = j <= i ? m[q] * ex2_fast(ci - cum2[j]) * delta[j] : 0.0f;
                        if (j == i) m[q] += dsk;
                    }
                }
            } else {
#pragma unroll
                for (int q = 0; q < 32; ++q) m[q] = 0.0f;
            }
            const uint32_t blk = (jb >> 1) * (kSsdQ * 128);
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
                uint4 hi, lo;
                split_bf16x2(m[pp * 8 + 0], m[pp * 8 + 1], hi.x, lo.x);
                split_bf16x2(m[pp * 8 + 2], m[pp * 8 + 3], hi.y, lo.y);
                split_bf16x2(m[pp * 8 + 4], m[pp * 8 + 5], hi.z, lo.z);
                split_bf16x2(m[pp * 8 + 6], m[pp * 8 + 7], hi.w, lo.w);
                const uint32_t off = blk + sw128_off(i, (jb & 1) * 4 + pp);
                *reinterpret_cast<uint4*>(bt + off) = hi;
                *reinterpret_cast<uint4*>(ht + off) = lo;
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // product 2: M X (hi and lo), K = Q = 128, N = P; x MN-major as copied
    bool x_loaded = true;
    if (g_ready && warp == 1 && elect_one_lane()) {
        x_done = x_issued && mbar_wait_bounded(&bars[3], 0, p.wait_limit);
        x_loaded = x_done;
        if (x_loaded) {
            constexpr uint32_t id_y = umma_idesc_bf16_mn(kSsdQ, kSsdP, false, true);
            const uint32_t mh = smem_addr(bt), ml = smem_addr(ht), xa = smem_addr(ct);
#pragma unroll
            for (int kk = 0; kk < kSsdQ / 16; ++kk) {
                const uint32_t mk = (kk >> 2) * (kSsdQ * 128) + (kk & 3) * 32;
                const uint64_t xdesc = umma_desc_sw128_mn(xa + kk * 2048, 0);
                umma_bf16(tmem + kSsdColDiag, umma_desc_sw128(mh + mk), xdesc, id_y, kk > 0 ? 1u : 0u);
                umma_bf16(tmem + kSsdColDiag, umma_desc_sw128(ml + mk), xdesc, id_y, 1u);
            }
            umma_commit(&bars[2]);
        }
    }
    const bool issued2 = __syncthreads_and(x_loaded) && g_ready;
    bool y_ok = false;
    if (issued2) y_ok = mbar_wait_bounded(&bars[2], 0, p.wait_limit);
    tc_fence_after();
    const bool y_ready = __syncthreads_and(y_ok);

    // y_i = (M X)_i + exp(cum_i) (C H_in^T)_i, gated by SiLU of the copied z
    // row; row i is staged over the x tile (free now), rows of 128 bytes with
    // their 16-byte pieces in the copies' swizzled order (piece q of row r at
    // q ^ (r % 8)), and the tile goes out by one bulk tensor store, which
    // writes no row past the sequence.
    if (y_ready) {
        const float e = ex2_fast(cum2[i]);
        const unsigned char* zrow = ct + kSsdQ * kSsdP * 2 + i * 128;
        unsigned char* yrow = ct + i * 128;
        {
            // this warpgroup's 32 output columns of row i
            float yo[32], yd[32];
            tmem_ld32(lane_base + kSsdColOff + wg * 32, yo);
            tmem_ld32(lane_base + kSsdColDiag + wg * 32, yd);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int piece = (wg * 4 + q) ^ (i & 7);
                float o[8];
#pragma unroll
                for (int e2 = 0; e2 < 8; ++e2) o[e2] = fmaf(e, yo[q * 8 + e2], yd[q * 8 + e2]);
                if (p.z) {
                    // SiLU(z) = hz + hz tanh(hz), hz = z / 2: one MUFU op
                    const uint4 zv = *reinterpret_cast<const uint4*>(zrow + piece * 16);
                    const float zf[8] = {bf16_lo(zv.x), bf16_hi(zv.x), bf16_lo(zv.y), bf16_hi(zv.y),
                                         bf16_lo(zv.z), bf16_hi(zv.z), bf16_lo(zv.w), bf16_hi(zv.w)};
#pragma unroll
                    for (int e2 = 0; e2 < 8; ++e2) {
                        const float hz = 0.5f * zf[e2];
                        o[e2] *= fmaf(hz, tanh_fast(hz), hz);
                    }
                }
                uint4 w;
                w.x = pack_bf16x2(o[0], o[1]);
                w.y = pack_bf16x2(o[2], o[3]);
                w.z = pack_bf16x2(o[4], o[5]);
                w.w = pack_bf16x2(o[6], o[7]);
                *reinterpret_cast<uint4*>(yrow + piece * 16) = w;
            }
        }
        // the staging writes, before the bulk store reads them
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            tma_store_3d(&tm_y, ct, h * kSsdP, static_cast<int>(t0), b);
            bulk_commit_group();
            bulk_wait_read_all();     // the store has read shared memory before the CTA ends
        }
    }

    if (!y_ready) {
        if (tid == 0) ssd_fail(p);
        // copies and products of this CTA finish before shared and tensor memory go away
        if (warp == 1 && elect_one_lane()) {
            if (!loaded) mbar_wait_bounded(&bars[0], 0, 1u << 20);
            if (issued1) mbar_wait_bounded(&bars[1], 0, 1u << 20);
            if (x_issued && !x_done) mbar_wait_bounded(&bars[3], 0, 1u << 20);
            if (issued2) mbar_wait_bounded(&bars[2], 0, 1u << 20);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, kSsdCols);
    }
}


// ---------------------------------------------------------------- one-token step (decode)
// The recurrence above for a single token per (head, sequence), in place on
// the state: with Delta = softplus(dt[h] + dt_bias[h]),
//     s[p,n] <- exp(Delta A[h]) s[p,n] + Delta x[p] B[n]
//     y[p]    = (sum_n C[n] s[p,n] + D[h] x[p]) SiLU(z[p])
// No product is dense enough for the tensor cores: each state entry is read
// once, updated and written back, so the step is bound by the state's HBM
// traffic (2 x 32 KB per head at P = 64, N = 128, fp32).  One CTA of 8 warps
// per (head, sequence); warp w holds state rows 8w .. 8w+7, lane l entries
// 4l .. 4l+3 of each (a warp's row is 512 contiguous bytes), all eight rows'
// loads in flight before the arithmetic.  A row's readout is a warp sum.
constexpr int kSsdDecThreads = 256;
constexpr int kSsdDecRows = kSsdP / (kSsdDecThreads / 32);    // state rows per warp
static_assert(kSsdDecRows == 8 && kSsdN == 4 * 32, "a warp covers 8 rows, a lane 4 entries of each");

struct SsdDecodeParams {
    const __nv_bfloat16* x;      // [B][H*P]
    const __nv_bfloat16* z;      // [B][H*P] or null (no gate)
    const __nv_bfloat16* dt;     // [B][H]
    const float* dt_bias;        // [H] or null
    const float* A;              // [H]
    const __nv_bfloat16* Bm;     // [B][G*N]
    const __nv_bfloat16* Cm;     // [B][G*N]
    const float* Dskip;          // [H] or null
    float* state;                // [B][H][P][N], updated in place
    __nv_bfloat16* y;            // [B][H*P]
    int H, G;
};

__global__ void __launch_bounds__(kSsdDecThreads)
ssd_state_update_kernel(const SsdDecodeParams p)
{
    const int h = blockIdx.x, b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = h / (p.H / p.G);
    const int64_t C = static_cast<int64_t>(p.H) * kSsdP;
    float4* st = reinterpret_cast<float4*>(p.state + ((static_cast<int64_t>(b) * p.H + h) * kSsdP +
                                                      warp * kSsdDecRows) * kSsdN) + lane;
    float4 s[kSsdDecRows];
#pragma unroll
    for (int r = 0; r < kSsdDecRows; ++r) s[r] = st[r * (kSsdN / 4)];

    const float v = __bfloat162float(p.dt[static_cast<int64_t>(b) * p.H + h]) + (p.dt_bias ? p.dt_bias[h] : 0.0f);
    const float dl = fmaxf(v, 0.0f) + log1pf(expf(-fabsf(v)));
    const float da = expf(dl * p.A[h]);
    const int64_t bc = (static_cast<int64_t>(b) * p.G + g) * kSsdN + 4 * lane;
    const uint2 braw = *reinterpret_cast<const uint2*>(p.Bm + bc);
    const uint2 craw = *reinterpret_cast<const uint2*>(p.Cm + bc);
    const float4 bv = make_float4(bf16_lo(braw.x), bf16_hi(braw.x), bf16_lo(braw.y), bf16_hi(braw.y));
    const float4 cv = make_float4(bf16_lo(craw.x), bf16_hi(craw.x), bf16_lo(craw.y), bf16_hi(craw.y));
    // x of the warp's 8 rows: one 16-byte load, the same for every lane
    const int64_t c0 = static_cast<int64_t>(b) * C + static_cast<int64_t>(h) * kSsdP + warp * kSsdDecRows;
    const uint4 xraw = *reinterpret_cast<const uint4*>(p.x + c0);
    const float xv[kSsdDecRows] = {bf16_lo(xraw.x), bf16_hi(xraw.x), bf16_lo(xraw.y), bf16_hi(xraw.y),
                                   bf16_lo(xraw.z), bf16_hi(xraw.z), bf16_lo(xraw.w), bf16_hi(xraw.w)};
    float mine = 0.0f;    // lane r < 8: the readout of row r
#pragma unroll
    for (int r = 0; r < kSsdDecRows; ++r) {
        const float u = dl * xv[r];
        s[r].x = fmaf(da, s[r].x, u * bv.x);
        s[r].y = fmaf(da, s[r].y, u * bv.y);
        s[r].z = fmaf(da, s[r].z, u * bv.z);
        s[r].w = fmaf(da, s[r].w, u * bv.w);
        st[r * (kSsdN / 4)] = s[r];
        float acc = fmaf(cv.x, s[r].x, fmaf(cv.y, s[r].y, fmaf(cv.z, s[r].z, cv.w * s[r].w)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
        if (lane == r) mine = acc;
    }
    if (lane < kSsdDecRows) {
        float xr = 0.0f;      // xv[lane], without a dynamic register index
#pragma unroll
        for (int r = 0; r < kSsdDecRows; ++r)
            if (lane == r) xr = xv[r];
        float yv = mine + (p.Dskip ? p.Dskip[h] : 0.0f) * xr;
        if (p.z) {
            const float zv = __bfloat162float(p.z[c0 + lane]);
            yv *= zv / (1.0f + expf(-zv));
        }
        p.y[c0 + lane] = __float2bfloat16_rn(yv);
    }
}

}  // namespace mm
