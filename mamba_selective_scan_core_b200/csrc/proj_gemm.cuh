// Projection GEMM on the fifth-generation tensor cores (tcgen05), for the
// dense products on either side of the selective scan: x_proj maps the conv
// output u_t (d_inner wide) to the low-rank step input and B_t, C_t; dt_proj
// maps the low-rank step input back to d_inner.  Both are
//
//     out[m, n] = sum_k A[m, k] * W[n, k]        A [M, K], W [N, K], bf16
//
// with fp32 accumulation: a weight stored one row per output feature, as a
// projection's weight is.
//
// One CTA computes NSUB adjacent 128 x BN tiles of `out` over a range of K
// (NSUB = 2 lets x_proj's 288 outputs, 2 x 144, share each tile of A, which
// is then read once; split-K gives tall, narrow products such as x_proj --
// 4096 x 288 x 8192 -- enough CTAs):
//   * warp 0 (one elected lane) streams 128 x 64 tiles of A and BN x 64 tiles
//     of W into a STAGES-deep shared-memory ring with 2-D tensor copies (TMA,
//     128-byte swizzle, no multicast);
//   * warp 1 (one elected lane) issues tcgen05.mma.kind::f16 (M 128, N BN,
//     K 16; four per 64-wide K tile) into an fp32 accumulator in tensor memory,
//     and releases each ring slot with tcgen05.commit once its MMAs are done;
//   * after the last MMA commits, all four warps read the accumulator with
//     tcgen05.ld (warp w owns rows 32w .. 32w+31, one row per thread) and
//     write it out: fp32 (a split-K partial) or bf16.  A bf16 output whose
//     tiles are whole 64-column boxes (and whose rows are 16-byte multiples)
//     is staged per warp in the ring's shared memory, free once the
//     accumulator is complete, as 32 x 64 boxes in the 128-byte swizzle, and
//     written by bulk tensor stores: whole lines, instead of one 16-byte piece
//     of 32 different rows per store instruction.
// Every wait on an mbarrier is bounded; a CTA that gives up sets the fault
// word, waits (bounded) for its own MMAs and copies, frees its tensor memory
// and exits.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "mixer_common.cuh"

namespace mm {

constexpr int kGemmBM = 128;      // rows of A per CTA (tcgen05 M)
constexpr int kGemmBK = 64;       // K per ring slot: one 128-byte swizzle atom of bf16
constexpr int kGemmThreads = 128;

struct GemmParams {
    void* out;              // [ksplit][M][N] fp32 partials, or [M][N] bf16 (row stride ldo elements)
    int64_t ldo;            // elements between rows of `out`
    int64_t split_stride;   // elements between split-K partials (fp32 output)
    int M, N, K;
    int k_tiles_per_split;  // 64-wide K tiles per CTA (blockIdx.z covers its own range)
    int tma_out;            // bf16 output written by bulk tensor stores through the output map
    unsigned wait_limit;    // tries per mbarrier wait before giving up
    unsigned long long* status;   // optional: [0] (epoch << 8) | code of a failure, [1] the call's epoch; or NULL
    unsigned long long status_epoch;
};

// ---------------------------------------------------------------- tcgen05 helpers
// Shared-memory matrix descriptor of a K-major tile written by a 128-byte
// swizzled tensor copy: rows of 128 bytes, 8-row groups 1024 bytes apart
// (stride byte offset), the leading offset unused for this layout, format
// version 1, layout type 2 (128-byte swizzle).  The tile must start on a
// 1024-byte boundary; advancing K by 16 bf16 advances the start by 32 bytes.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_byte_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_byte_addr >> 4) & 0x3FFF);          // start address
    d |= static_cast<uint64_t>(1) << 16;                                  // leading byte offset (16 B)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;                          // stride byte offset
    d |= static_cast<uint64_t>(1) << 46;                                  // version
    d |= static_cast<uint64_t>(2) << 61;                                  // 128-byte swizzle
    return d;
}

// Instruction descriptor of tcgen05.mma.kind::f16: bf16 A and B, both
// K-major, fp32 accumulator, M x N.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int m, int n) {
    return (1u << 4)                                   // accumulator format: f32
         | (1u << 7)                                   // A format: bf16
         | (1u << 10)                                  // B format: bf16
         | (static_cast<uint32_t>(n >> 3) << 17)       // N / 8
         | (static_cast<uint32_t>(m >> 4) << 24);      // M / 16
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n"
                 :: "r"(smem_addr(dst_smem)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" :: "r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
// D (tensor memory) = A * B^T (+ D when accumulate): both operands in shared memory
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
        :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
// arrive on `bar` once every tcgen05.mma this thread issued so far has completed
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n"
                 :: "r"(smem_addr(bar)) : "memory");
}
// 32 consecutive fp32 columns of this thread's row (lane) of tensor memory
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 fp32 columns of this thread's row of tensor memory, without waiting:
// the registers are valid after tmem_wait_ld
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }

// 2-D tiled bulk tensor copy shared -> global (a store), in this thread's
// bulk group; rows and columns outside the tensor are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];\n"
                 :: "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(src)) : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;\n" ::: "memory"); }
// every bulk store this thread committed has read its shared-memory source
// (the writes themselves complete before the grid does)
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory"); }

// 2-D tiled bulk tensor copy global -> shared, completion on `bar`.  No multicast.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n"
        :: "r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(bar))
        : "memory");
}

template <int BN, int NSUB = 1>
struct GemmLayout {
    static constexpr int a_bytes = kGemmBM * kGemmBK * 2;       // 16 KB, a multiple of 1024
    static constexpr int b_bytes = BN * kGemmBK * 2;            // BN x 128 B per sub-tile
    static constexpr int stage_bytes = a_bytes + NSUB * b_bytes;
    static constexpr int acc_cols = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;   // per sub-tile
    static constexpr int tmem_cols = NSUB * acc_cols;
    // ring, then full[STAGES], empty[STAGES], acc barrier and the tensor-memory address
    static constexpr int smem_bytes(int stages) { return 1024 + stages * stage_bytes + (2 * stages + 2) * 8 + 16; }
};

// OUT_BF16: write bf16 rows (no split-K); else fp32 split-K partials.
template <int BN, int NSUB, int STAGES, bool OUT_BF16>
__global__ void __launch_bounds__(kGemmThreads, 1)
proj_gemm_kernel(const GemmParams p, const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
                 const __grid_constant__ CUtensorMap tm_out)
{
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "tcgen05 N for M = 128");
    static_assert(GemmLayout<BN>::b_bytes % 1024 == 0, "ring slots stay 1024-byte aligned");
    static_assert(NSUB == 1 || NSUB == 2, "one or two sub-tiles");
    using Lay = GemmLayout<BN, NSUB>;
    extern __shared__ __align__(1024) unsigned char gsm_raw[];
    // the swizzled tiles must start on 1024-byte boundaries
    unsigned char* gsm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(gsm + STAGES * Lay::stage_bytes);
    uint64_t* empty = full + STAGES;
    uint64_t* accb = empty + STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accb + 2);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    // the call's epoch, in the status word's second half (written from the
    // device, so that a captured call records no host copy)
    if (p.status && tid == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) p.status[1] = p.status_epoch;
    const int m0 = blockIdx.x * kGemmBM;
    const int n0 = blockIdx.y * BN * NSUB;
    const int kt0 = blockIdx.z * p.k_tiles_per_split;
    const int k_tiles_total = (p.K + kGemmBK - 1) / kGemmBK;
    const int nkt = max(0, min(p.k_tiles_per_split, k_tiles_total - kt0));

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accb, 1);
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc(tmem_slot, Lay::tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool ok = true;
    constexpr uint32_t idesc = umma_idesc_bf16(kGemmBM, BN);
    const unsigned tx_bytes = Lay::stage_bytes;
    int issued = 0;     // tile copies issued (producer thread), for the bounded drain on failure

    if (warp == 0) {
        if (elect_one_lane()) {
            for (int k = 0; k < nkt; ++k) {
                const int s = k % STAGES;
                // the slot is free once the MMAs that read it have completed
                if (!mbar_wait_bounded(&empty[s], static_cast<unsigned>(((k / STAGES) & 1) ^ 1), p.wait_limit)) {
                    ok = false;
                    break;
                }
                unsigned char* st = gsm + s * Lay::stage_bytes;
                mbar_arrive_expect_tx(&full[s], tx_bytes);
                const int kc = (kt0 + k) * kGemmBK;
                tma_load_2d(st, &tm_a, kc, m0, &full[s]);
#pragma unroll
                for (int j = 0; j < NSUB; ++j)
                    tma_load_2d(st + Lay::a_bytes + j * Lay::b_bytes, &tm_w, kc, n0 + j * BN, &full[s]);
                ++issued;
            }
        }
    } else if (warp == 1) {
        if (elect_one_lane()) {
            for (int k = 0; k < nkt; ++k) {
                const int s = k % STAGES;
                if (!mbar_wait_bounded(&full[s], static_cast<unsigned>((k / STAGES) & 1), p.wait_limit)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_base = smem_addr(gsm + s * Lay::stage_bytes);
                const uint32_t b_base = a_base + Lay::a_bytes;
#pragma unroll
                for (int kk = 0; kk < kGemmBK / 16; ++kk)
#pragma unroll
                    for (int j = 0; j < NSUB; ++j)
                        umma_bf16(tmem + j * Lay::acc_cols, umma_desc_sw128(a_base + kk * 32),
                                  umma_desc_sw128(b_base + j * Lay::b_bytes + kk * 32), idesc,
                                  (k > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&empty[s]);
            }
            // the accumulator is complete once every MMA issued above has finished
            umma_commit(accb);
        }
    }
    // a failure anywhere in the CTA stops the epilogue
    const bool all_ok = __syncthreads_and(ok);
    if (!all_ok) {
        if (tid == 0) {
            atomicOr(&g_mm_fault, 1u);
            if (p.status) atomicExch(p.status, (p.status_epoch << 8) | 1ull);
        }
    }
    // wait (bounded) for the MMAs to finish before tensor memory is read or freed
    const bool acc_ready = mbar_wait_bounded(accb, 0, all_ok ? p.wait_limit : (1u << 20));
    tc_fence_after();

    // staged bf16 output: 128 rows x BN columns in the ring (free: every MMA
    // that read it has completed); warp w's 32 rows of 64-column box bx at
    // (bx * 4 + w) * 4 KB, 16-byte pieces swizzled by row as the map expects
    constexpr bool kStaged = OUT_BF16 && NSUB == 1 && BN % 64 == 0 &&
                             STAGES * Lay::stage_bytes >= kGemmBM * BN * 2;
    if (kStaged && p.tma_out && all_ok && acc_ready) {
        const int r = tid & 31;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        // a box's 64 columns per round: two tensor-memory loads, one wait
#pragma unroll 1
        for (int bx = 0; bx < BN / 64; ++bx) {
            uint32_t u[2][32];
            tmem_ld32_async(lane_base + bx * 64, u[0]);
            tmem_ld32_async(lane_base + bx * 64 + 32, u[1]);
            tmem_wait_ld();
            unsigned char* slab = gsm + (bx * 4 + warp) * 4096;
#pragma unroll
            for (int piece = 0; piece < 8; ++piece) {     // 16-byte piece of the 128-byte box row
                const uint32_t* q = u[piece >> 2] + 8 * (piece & 3);
                float v[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = nkt == 0 ? 0.0f : __uint_as_float(q[i]);
                uint4 w;
                w.x = pack_bf16x2(v[0], v[1]);
                w.y = pack_bf16x2(v[2], v[3]);
                w.z = pack_bf16x2(v[4], v[5]);
                w.w = pack_bf16x2(v[6], v[7]);
                *reinterpret_cast<uint4*>(slab + (r >> 3) * 1024 + (r & 7) * 128 + ((piece ^ (r & 7)) << 4)) = w;
            }
        }
        // the generic-proxy writes above, before the bulk stores read them
        fence_proxy_async_smem();
        __syncwarp();
        if (elect_one_lane()) {
#pragma unroll 1
            for (int bx = 0; bx < BN / 64; ++bx)
                tma_store_2d(&tm_out, gsm + (bx * 4 + warp) * 4096, n0 + bx * 64, m0 + warp * 32);
            bulk_commit_group();
            // the stores have read shared memory before the CTA ends
            bulk_wait_read_all();
        }
        __syncwarp();
    } else if (all_ok && acc_ready) {
        const int row = m0 + warp * 32 + (tid & 31);
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        // sub-tile j's accumulator sits at column j * acc_cols; its BN columns
        // are read in chunks of 32 (the last one partial when BN is not a
        // multiple of 32) and written at output column n0 + j * BN + c0
#pragma unroll 1
        for (int jc = 0; jc < NSUB * ((BN + 31) / 32); ++jc) {
            const int j = jc / ((BN + 31) / 32);
            const int c0 = (jc - j * ((BN + 31) / 32)) * 32;
            const int nb = n0 + j * BN;      // first output column of this sub-tile
            float v[32];
            tmem_ld32(lane_base + j * Lay::acc_cols + c0, v);
            if (nkt == 0) {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.0f;
            }
            if (row < p.M) {
                // columns of this chunk inside both the tile (BN need not be a
                // multiple of 32) and the matrix
                const int ncol = min(min(32, BN - c0), p.N - (nb + c0));
                if (ncol > 0) {
                    if constexpr (OUT_BF16) {
                        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(row) * p.ldo + nb + c0;
                        if (ncol == 32) {
#pragma unroll
                            for (int i = 0; i < 32; i += 8) {
                                uint4 w;
                                w.x = pack_bf16x2(v[i], v[i + 1]);
                                w.y = pack_bf16x2(v[i + 2], v[i + 3]);
                                w.z = pack_bf16x2(v[i + 4], v[i + 5]);
                                w.w = pack_bf16x2(v[i + 6], v[i + 7]);
                                *reinterpret_cast<uint4*>(o + i) = w;
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (i < ncol) o[i] = __float2bfloat16_rn(v[i]);
                        }
                    } else {
                        float* o = static_cast<float*>(p.out) + blockIdx.z * p.split_stride +
                                   static_cast<int64_t>(row) * p.ldo + nb + c0;
                        if (ncol == 32) {
#pragma unroll
                            for (int i = 0; i < 32; i += 4)
                                *reinterpret_cast<float4*>(o + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (i < ncol) o[i] = v[i];
                        }
                    }
                }
            }
        }
    } else if (!acc_ready && tid == 0) {
        atomicOr(&g_mm_fault, 1u);
        if (p.status) atomicExch(p.status, (p.status_epoch << 8) | 1ull);
    }
    // in a failed CTA, the copies the producer issued land before shared memory
    // goes away: each slot's latest copy completes its latest phase
    if (!all_ok && warp == 0 && elect_one_lane()) {
        for (int j = max(0, issued - STAGES); j < issued; ++j)
            mbar_wait_bounded(&full[j % STAGES], static_cast<unsigned>((j / STAGES) & 1), 1u << 20);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, Lay::tmem_cols);
    }
}

}  // namespace mm
