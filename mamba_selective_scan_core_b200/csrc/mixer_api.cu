// Host side of the C ABI declared in include/mamba_mixer.h: argument
// validation (before anything is launched), launch-shape selection and the
// launches themselves.  No allocation.  The only state is the device fault
// word, the fixed scratch array of mamba_mixer_fwd_noalloc with its
// per-device address, and the tensor-map encoder's entry point.
#include <algorithm>
#include <cudaTypedefs.h>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "mamba_mixer.h"
#include "mixer_decode.cuh"
#include "mixer_prefill.cuh"

namespace {

using mm::PrefillLayout;
using mm::PrefillParams;

constexpr int kTile = 32;
constexpr int kMaxThreads = 128;
constexpr int kSmemBudget = 200 * 1024;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Span {
    uintptr_t lo = 0, hi = 0;   // [lo, hi); empty when lo == hi
};
Span span(const void* p, int64_t bytes) {
    Span s;
    if (p && bytes > 0) {
        s.lo = reinterpret_cast<uintptr_t>(p);
        s.hi = s.lo + static_cast<uintptr_t>(bytes);
    }
    return s;
}
bool overlaps(const Span& a, const Span& b) { return a.lo < a.hi && b.lo < b.hi && a.lo < b.hi && b.lo < a.hi; }

// a * b with overflow detection on non-negative operands
bool mul_ok(int64_t a, int64_t b, int64_t* out) {
    if (a < 0 || b < 0) return false;
    if (a != 0 && b > INT64_MAX / a) return false;
    *out = a * b;
    return true;
}

// Sequence lengths the forward's bulk tensor copies can address: token
// coordinates are 32-bit, and the copy engine takes strides below 2^40 bytes,
// which bounds one sequence's xz rows (seqlen x 2 d_inner elements).  Longer
// sequences are run as several calls with the state carried.
constexpr int64_t kMaxSeqlen = int64_t(1) << 30;
bool seqlen_ok(int64_t seqlen, int64_t d_inner, int64_t es) {
    return seqlen <= kMaxSeqlen && seqlen * 2 * d_inner * es < (int64_t(1) << 40);
}

mm_status check_device(int* sm_count) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return MM_ERR_DEVICE; }
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return MM_ERR_DEVICE;
    }
    if (major != 10) return MM_ERR_DEVICE;
    return MM_OK;
}

// Launch plan of a forward call: time chunks and the workspace they need.
// A pure function of the sizes (and of the MAMBA_MIXER_CHUNKS tuning
// variable), so that mamba_mixer_workspace_size() and the call agree.
struct FwdPlan {
    int chunks = 1;
    int64_t chunk_len = 0;
    size_t ws_bytes = 0;
};

constexpr int kPlanSMs = 148;            // B200: 2 dies x 74 SMs
constexpr int kWarpsPerSM = 4 * MM_FWD_MIN_BLOCKS;   // resident warps per SM at the forward's register use
constexpr int kMinChunkTiles = 4;        // shortest chunk worth a summary pass
constexpr int kMaxChunks = 16;

int env_int(const char* name, int lo, int hi) {
    if (const char* e = std::getenv(name)) {
        const int v = std::atoi(e);
        if (v >= lo && v <= hi) return v;
    }
    return 0;
}

// Tries per wait on a bulk copy (each try waits a bounded time in hardware):
// about a second by default; MAMBA_MIXER_WAIT_LIMIT overrides it (tests use 0
// to make the wait give up at once).
unsigned copy_wait_limit() {
    if (const char* e = std::getenv("MAMBA_MIXER_WAIT_LIMIT")) {
        char* end = nullptr;
        const long v = std::strtol(e, &end, 10);
        if (end != e && v >= 0 && v <= (1L << 30)) return static_cast<unsigned>(v);
    }
    return 1u << 20;
}

// Time chunks.  More chunks put more warps on the SMs but add a summary pass
// over (K-1)/K of the tokens, so K minimises a measured cost model: a pass
// takes about (tokens per chunk) x (time of its busiest SM), an SM running
// 8 warps (two CTAs) taking ~1.85x as long as one running 4, and a summary
// token costing ~0.55 of a full-pass token (B200 measurements of both
// kernels), among splits that fit one wave.  It picks 9 chunks for one
// 8192-channel sequence and a single chunk once a batch fills the SMs on
// its own.
double busiest_sm(int64_t warps) {
    const int64_t m = (warps + kPlanSMs - 1) / kPlanSMs;        // warps on the busiest SM
    const int64_t waves = m / kWarpsPerSM, rest = m % kWarpsPerSM;
    return 1.85 * static_cast<double>(waves) + (rest == 0 ? 0.0 : rest * 2 <= kWarpsPerSM ? 1.0 : 1.85);
}

FwdPlan plan_fwd(int64_t batch, int64_t seqlen, int64_t d_inner) {
    FwdPlan pl;
    const int64_t warps = std::max<int64_t>(1, batch * ((d_inner / 2 + 31) / 32));   // per chunk
    const int64_t tiles = std::max<int64_t>(1, (seqlen + kTile - 1) / kTile);
    auto chunk_tiles = [&](int64_t k) { return (tiles + k - 1) / k; };
    int64_t k = 1;
    if (const int forced = env_int("MAMBA_MIXER_CHUNKS", 1, 1 << 20)) {
        k = std::min<int64_t>(forced, tiles);
    } else {
        double best = 0.0;
        const int64_t kmax = std::min<int64_t>(kMaxChunks, std::max<int64_t>(1, tiles / kMinChunkTiles));
        for (int64_t c = 1; c <= kmax; ++c) {
            const int64_t ct = chunk_tiles(c);
            const int64_t chunks = (tiles + ct - 1) / ct;            // chunks the split really makes
            // a split stays within one wave of resident warps (the model does not
            // charge what grows with the chunk count: carry chains, pipeline fills)
            if (chunks > 1 && chunks * warps > static_cast<int64_t>(kPlanSMs) * kWarpsPerSM) break;
            const double cost = static_cast<double>(ct) *
                                (busiest_sm(chunks * warps) + (chunks > 1 ? 0.55 * busiest_sm((chunks - 1) * warps) : 0.0));
            if (c == 1 || cost < best) { best = cost; k = c; }
        }
    }
    pl.chunk_len = chunk_tiles(k) * kTile;
    pl.chunks = static_cast<int>(seqlen > 0 ? (seqlen + pl.chunk_len - 1) / pl.chunk_len : 1);
    if (pl.chunks > 1)
        pl.ws_bytes = static_cast<size_t>(pl.chunks - 1) * batch * d_inner * (16 + 1) * sizeof(float);
    return pl;
}

// ---------------------------------------------------------------- tensor maps
// The driver's tensor-map encoder, fetched through the runtime (no link
// against libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        cudaGetLastError();
    });
    return fn;
}

struct TensorMaps {
    CUtensorMap x, z, dt, b, c;
};

// 3-D map over a [batch][rows][cols] tensor with a [1][box_rows][box_cols] box.
bool encode_3d(CUtensorMap* m, const void* base, bool bf16, int64_t cols, int64_t rows, int64_t batch,
               int box_cols, int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const int64_t es = bf16 ? 2 : 4;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                                static_cast<cuuint64_t>(batch)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols * es), static_cast<cuuint64_t>(rows * cols * es)};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
               const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T>
bool make_maps(const PrefillParams& p, int64_t batch, TensorMaps* m) {
    std::memset(m, 0, sizeof(*m));
    if (p.L == 0) return true;                 // no tiles: the maps are never read
    constexpr bool bf16 = sizeof(T) == 2;
    const int boxc = p.octets * 8;
    return encode_3d(&m->x, p.xz, bf16, 2 * int64_t(p.D), p.L, batch, boxc, kTile + mm::kHalo) &&
           encode_3d(&m->z, p.xz, bf16, 2 * int64_t(p.D), p.L, batch, boxc, kTile) &&
           encode_3d(&m->dt, p.dt, bf16, p.D, p.L, batch, boxc, kTile) &&
           encode_3d(&m->b, p.Bm, bf16, 16, p.L, batch, 16, kTile) &&
           encode_3d(&m->c, p.Cm, bf16, 16, p.L, batch, 16, kTile);
}

// `dependent`: launch as a programmatic dependent of the kernel before it in
// the stream (the summary pass of the same call), see mixer_fwd_kernel.
template <typename T, typename M, int STAGES, bool SUMMARY>
cudaError_t launch_prefill(const PrefillParams& p, int64_t batch, int chunks, int threads, bool dependent,
                           cudaStream_t s) {
    auto kern = mm::mixer_fwd_kernel<T, M, kTile, STAGES, SUMMARY>;
    TensorMaps maps;
    if (!make_maps<T>(p, batch, &maps)) return cudaErrorInvalidValue;
    const int smem = PrefillLayout<T>::smem_bytes(kTile, STAGES, p.octets);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(batch * p.ctas_per_seq), static_cast<unsigned>(chunks));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kern, p, maps.x, maps.z, maps.dt, maps.b, maps.c);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// Octets per CTA (4 threads per octet) and copy-ring depth.  Every warp of
// a pass does the same work, so the pass takes about one warp's time per
// wave: pick the shape with the fewest waves, counting how many CTAs an SM
// holds under both its register file (8 warps at the forward's register use)
// and its shared memory; among equals prefer the wider CTA (B/C staging is
// shared by a CTA's channels), then the deeper ring.
constexpr int kSmemPerSM = 227 * 1024;

template <typename T>
int ring_depth(int oct) {
    for (int st = 4; st >= 2; --st)
        if (PrefillLayout<T>::smem_bytes(kTile, st, oct) <= kSmemBudget) return st;
    return 0;
}

template <typename T>
int shape_ctas(PrefillParams& p, int64_t batch, int64_t chunks, int sm_count, int* threads) {
    const int64_t octets_per_seq = p.D / 8;
    // a copy box spans at most 256 channels: 32 octets
    const int max_oct = static_cast<int>(std::min<int64_t>({kMaxThreads / 4, 32, octets_per_seq}));
    int64_t best_waves = INT64_MAX;
    int best = 1, best_stages = 2;
    for (int oct = 1; oct <= max_oct; ++oct) {
        const int64_t per_seq = (octets_per_seq + oct - 1) / oct;
        if (per_seq * oct - octets_per_seq >= oct) continue;        // same CTA count as a smaller oct
        const int warps = (oct * 4 + 31) / 32;
        for (int st = ring_depth<T>(oct); st >= 2; --st) {
            const int smem = PrefillLayout<T>::smem_bytes(kTile, st, oct);
            const int per_sm = std::max(1, std::min(kWarpsPerSM / warps, kSmemPerSM / smem));
            const int64_t slots = static_cast<int64_t>(sm_count) * per_sm;
            const int64_t waves = (batch * per_seq * chunks + slots - 1) / slots;
            if (waves < best_waves || (waves == best_waves && (oct > best || (oct == best && st > best_stages)))) {
                best_waves = waves; best = oct; best_stages = st;
            }
        }
    }
    const int64_t ctas = (octets_per_seq + best - 1) / best;
    p.octets = static_cast<int>((octets_per_seq + ctas - 1) / ctas);
    p.ctas_per_seq = static_cast<int>(ctas);
    *threads = ((p.octets * 4) + 31) / 32 * 32;
    return std::min(best_stages, std::max(2, ring_depth<T>(p.octets)));
}

template <typename T, typename M, bool SUMMARY>
cudaError_t launch_pass(PrefillParams p, int64_t batch, int chunks, int sm_count, bool dependent, cudaStream_t s) {
    int threads = 0;
    const int stages = shape_ctas<T>(p, batch, chunks, sm_count, &threads);
    if (stages >= 4) return launch_prefill<T, M, 4, SUMMARY>(p, batch, chunks, threads, dependent, s);
    if (stages == 3) return launch_prefill<T, M, 3, SUMMARY>(p, batch, chunks, threads, dependent, s);
    return launch_prefill<T, M, 2, SUMMARY>(p, batch, chunks, threads, dependent, s);
}

template <typename T, typename M>
cudaError_t dispatch_prefill(PrefillParams p, int64_t batch, const FwdPlan& pl, int sm_count, cudaStream_t s) {
    p.chunk_len = pl.chunk_len;
    p.n_chunks = pl.chunks;
    // The summary pass is launched normally: it starts after everything
    // before it in the stream, the producers of the inputs included.  The
    // full pass follows it as a programmatic dependent; its CTAs read the
    // inputs freely (they were complete before the summary pass started) and
    // wait for the summary grid before reading its results.
    if (pl.chunks > 1) {
        cudaError_t e = launch_pass<T, M, true>(p, batch, pl.chunks - 1, sm_count, false, s);
        if (e != cudaSuccess) return e;
    }
    return launch_pass<T, M, false>(p, batch, pl.chunks, sm_count, pl.chunks > 1, s);
}

// ---------------------------------------------------------------- host-memory forward
// Piece plan of mamba_mixer_fwd_host: the sequence is cut into about
// kHostPieces pieces (whole tiles, at least kHostMinPiece tokens) and the
// device workspace holds two staging slots, two carried states (ping-pong)
// and the piece forward's own scratch, each region 256-byte aligned.  What
// follows the last input copy -- the last piece's forward and the copy back
// of its y -- is the call's tail, so a last piece of at least kHostMinPiece
// tokens is cut once more, in two.
constexpr int64_t kHostPieces = 8;
constexpr int64_t kHostMinPiece = 256;

struct HostPlan {
    int64_t piece = 0, pieces = 0;
    int64_t head = 0;     // pieces 0..head-1 hold `piece` tokens each
    int64_t tail1 = 0;    // the rest: one piece, or (tail1 > 0) tail1 tokens then the remainder
    size_t off_dt = 0, off_b = 0, off_c = 0, off_y = 0, slot = 0;   // within a staging slot
    size_t carry_h = 0, carry = 0;                                  // within a carried state
    size_t fwd_ws = 0, total = 0;
};

size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

// First token and length of piece i of a plan over `seqlen` tokens.
void piece_range(const HostPlan& hp, int64_t i, int64_t seqlen, int64_t* t0, int64_t* n) {
    const int64_t tail = hp.head * hp.piece;
    if (i < hp.head) { *t0 = i * hp.piece; *n = hp.piece; }
    else if (hp.tail1 == 0) { *t0 = tail; *n = seqlen - tail; }
    else if (i == hp.head) { *t0 = tail; *n = hp.tail1; }
    else { *t0 = tail + hp.tail1; *n = seqlen - tail - hp.tail1; }
}

HostPlan plan_host(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t es) {
    HostPlan hp;
    int64_t piece = (seqlen + kHostPieces - 1) / kHostPieces;
    piece = (piece + kTile - 1) / kTile * kTile;
    piece = std::max(piece, kHostMinPiece);
    hp.piece = std::max<int64_t>(1, std::min(piece, seqlen));
    hp.head = seqlen > 0 ? (seqlen + hp.piece - 1) / hp.piece - 1 : 0;   // L = 0: one empty piece
    const int64_t rest = seqlen - hp.head * hp.piece;
    hp.tail1 = rest >= kHostMinPiece ? ((rest + 1) / 2 + kTile - 1) / kTile * kTile : 0;
    hp.pieces = hp.head + (hp.tail1 > 0 ? 2 : 1);
    const size_t tok = static_cast<size_t>(batch) * static_cast<size_t>(hp.piece);
    const size_t D = static_cast<size_t>(d_inner), e = static_cast<size_t>(es);
    hp.off_dt = align256(tok * 2 * D * e);
    hp.off_b = hp.off_dt + align256(tok * D * e);
    hp.off_c = hp.off_b + align256(tok * 16 * e);
    hp.off_y = hp.off_c + align256(tok * 16 * e);
    hp.slot = hp.off_y + align256(tok * D * e);
    hp.carry_h = align256(static_cast<size_t>(batch) * D * 16 * 4);
    hp.carry = hp.carry_h + align256(static_cast<size_t>(batch) * D * 3 * e);
    // the scratch must fit the plan of every piece length used
    size_t ws = plan_fwd(batch, hp.tail1 > 0 ? hp.tail1 : rest, d_inner).ws_bytes;
    if (hp.head > 0) ws = std::max(ws, plan_fwd(batch, hp.piece, d_inner).ws_bytes);
    if (hp.tail1 > 0) ws = std::max(ws, plan_fwd(batch, rest - hp.tail1, d_inner).ws_bytes);
    hp.fwd_ws = align256(ws);
    hp.total = 2 * hp.slot + 2 * hp.carry + hp.fwd_ws;
    return hp;
}

// Events of one mamba_mixer_fwd_host call, destroyed when it returns (the
// driver releases an event still pending once it completes).
struct HostEvents {
    cudaEvent_t ev[8] = {};
    int n = 0;
    cudaEvent_t make() {
        cudaEvent_t e = nullptr;
        if (n < 8 && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess) ev[n++] = e;
        return e;
    }
    ~HostEvents() {
        for (int i = 0; i < n; ++i) cudaEventDestroy(ev[i]);
    }
};

}  // namespace

// Scratch of mamba_mixer_fwd_noalloc: one fixed array per device in the
// library's device image, for callers that cannot allocate.  Host code only
// ever passes its device address (looked up per device, below) to kernels.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MAMBA_MIXER_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 256;

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (with that device current) and kept.
mm_status noalloc_scratch(void** out) {
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return MM_ERR_DEVICE; }
    if (dev < 0 || dev >= kMaxDevices) return MM_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return MM_ERR_CUDA;
        }
        addr[dev] = p;
    }
    *out = addr[dev];
    return MM_OK;
}

}  // namespace

extern "C" {

int mamba_mixer_abi_version(void) { return MAMBA_MIXER_ABI_VERSION; }

const char* mamba_status_string(mm_status status) {
    switch (status) {
        case MM_OK: return "ok";
        case MM_ERR_NULL: return "a required pointer is NULL";
        case MM_ERR_SHAPE: return "invalid size (negative, zero where not allowed, or too large)";
        case MM_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case MM_ERR_DTYPE: return "unknown activation dtype";
        case MM_ERR_ALIAS: return "an output overlaps an input or another output";
        case MM_ERR_UNSUPPORTED: return "unsupported size (need d_state == 16, d_conv == 4, d_inner % 8 == 0)";
        case MM_ERR_CUDA: return "CUDA runtime error at launch";
        case MM_ERR_DEVICE: return "no usable sm_100 device is current";
        case MM_ERR_WORKSPACE: return "workspace missing or smaller than mamba_mixer_workspace_size()";
        case MM_ERR_TIMEOUT: return "a kernel gave up waiting for its bulk copies (see mamba_mixer_fault_status)";
        case MM_ERR_SCRATCH_LIMIT:
            return "sizes need more scratch than mamba_mixer_fwd_noalloc's built-in 8 MiB; pass a workspace to "
                   "mamba_mixer_fwd instead";
    }
    return "unknown status";
}

mm_status mamba_mixer_fault_status(int reset) {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, mm::g_mm_fault, sizeof(v)) != cudaSuccess) { cudaGetLastError(); return MM_ERR_CUDA; }
    if (reset && v) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(mm::g_mm_fault, &zero, sizeof(zero)) != cudaSuccess) { cudaGetLastError(); return MM_ERR_CUDA; }
    }
    return v ? MM_ERR_TIMEOUT : MM_OK;
}

size_t mamba_mixer_workspace_size(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state,
                                  int64_t d_conv, mm_dtype act) {
    if ((act != MM_F32 && act != MM_BF16) || batch <= 0 || seqlen <= 0 || d_inner <= 0 || d_state != 16 ||
        d_conv != 4 || d_inner % 8 != 0 || d_inner > (1 << 24) || batch > (1 << 24) ||
        !seqlen_ok(seqlen, d_inner, act == MM_F32 ? 4 : 2))
        return 0;
    return plan_fwd(batch, seqlen, d_inner).ws_bytes;
}

mm_status mamba_mixer_fwd(const void* xz, const float* conv_w, const float* conv_b,
                          const void* dt, const float* dt_bias, const float* A,
                          const void* Bm, const void* Cm, const float* Dskip,
                          const float* h0, const void* conv_state_in,
                          void* y, float* h_last, void* conv_state_out,
                          int64_t batch, int64_t seqlen, int64_t d_inner,
                          int64_t d_state, int64_t d_conv, mm_dtype act,
                          void* workspace, size_t workspace_bytes, void* stream)
{
    if (act != MM_F32 && act != MM_BF16) return MM_ERR_DTYPE;
    if (batch < 0 || seqlen < 0 || d_inner <= 0 || d_state <= 0 || d_conv <= 0) return MM_ERR_SHAPE;
    if (d_state != 16 || d_conv != 4 || d_inner % 8 != 0) return MM_ERR_UNSUPPORTED;
    if (d_inner > (1 << 24) || batch > (1 << 24)) return MM_ERR_SHAPE;
    const int64_t es = act == MM_F32 ? 4 : 2;
    if (!seqlen_ok(seqlen, d_inner, es)) return MM_ERR_SHAPE;
    int64_t tokens, xz_bytes, dt_bytes, bc_bytes, st_bytes;
    if (!mul_ok(batch, seqlen, &tokens) || !mul_ok(tokens, 2 * d_inner * es, &xz_bytes) ||
        !mul_ok(tokens, d_inner * es, &dt_bytes) || !mul_ok(tokens, d_state * es, &bc_bytes) ||
        !mul_ok(batch, d_inner * d_state * 4, &st_bytes))
        return MM_ERR_SHAPE;
    const int64_t cs_bytes = batch * d_inner * (d_conv - 1) * es;
    if (batch == 0) return MM_OK;

    // required pointers
    if (!conv_w || !dt_bias || !A || !h_last || !conv_state_out) return MM_ERR_NULL;
    if (seqlen > 0 && (!xz || !dt || !Bm || !Cm || !y)) return MM_ERR_NULL;
    const void* all[] = {xz, conv_w, conv_b, dt, dt_bias, A, Bm, Cm, Dskip, h0, conv_state_in,
                         y, h_last, conv_state_out};
    for (const void* q : all)
        if (q && !aligned16(q)) return MM_ERR_ALIGN;

    const Span in[] = {span(xz, xz_bytes), span(conv_w, d_inner * d_conv * 4), span(conv_b, d_inner * 4),
                       span(dt, dt_bytes), span(dt_bias, d_inner * 4), span(A, d_inner * d_state * 4),
                       span(Bm, bc_bytes), span(Cm, bc_bytes), span(Dskip, d_inner * 4),
                       span(h0, st_bytes), span(conv_state_in, cs_bytes)};
    const Span out[] = {span(y, dt_bytes), span(h_last, st_bytes), span(conv_state_out, cs_bytes)};
    for (const Span& o : out)
        for (const Span& i : in)
            if (overlaps(o, i)) return MM_ERR_ALIAS;
    if (overlaps(out[0], out[1]) || overlaps(out[0], out[2]) || overlaps(out[1], out[2])) return MM_ERR_ALIAS;

    const FwdPlan pl = plan_fwd(batch, seqlen, d_inner);
    if (pl.ws_bytes > 0) {
        if (!workspace || workspace_bytes < pl.ws_bytes) return MM_ERR_WORKSPACE;
        if (!aligned16(workspace)) return MM_ERR_ALIGN;
        const Span ws = span(workspace, static_cast<int64_t>(pl.ws_bytes));
        for (const Span& i : in)
            if (overlaps(ws, i)) return MM_ERR_ALIAS;
        for (const Span& o : out)
            if (overlaps(ws, o)) return MM_ERR_ALIAS;
    }

    int sm_count = 0;
    if (mm_status st = check_device(&sm_count); st != MM_OK) return st;

    PrefillParams p{};
    p.xz = xz; p.conv_w = conv_w; p.conv_b = conv_b; p.dt = dt; p.dt_bias = dt_bias; p.A = A;
    p.Bm = Bm; p.Cm = Cm; p.Dskip = Dskip; p.h0 = h0; p.cs_in = conv_state_in;
    p.y = y; p.h_last = h_last; p.cs_out = conv_state_out;
    p.L = seqlen;
    p.D = static_cast<int>(d_inner);
    p.batch = static_cast<int>(batch);
    p.wait_limit = copy_wait_limit();
    p.ws_state = static_cast<float*>(workspace);
    p.ws_lsum = pl.ws_bytes ? p.ws_state + static_cast<int64_t>(pl.chunks - 1) * batch * d_inner * 16 : nullptr;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = act == MM_BF16 ? dispatch_prefill<__nv_bfloat16, mm::MathFast>(p, batch, pl, sm_count, s)
                                   : dispatch_prefill<float, mm::MathExact>(p, batch, pl, sm_count, s);
    if (e != cudaSuccess) { cudaGetLastError(); return MM_ERR_CUDA; }
    return MM_OK;
}

mm_status mamba_state_update(const void* x, const void* z, const void* dt,
                             const float* conv_w, const float* conv_b,
                             const float* dt_bias, const float* Dskip, const float* A,
                             const void* Bm, const void* Cm,
                             float* ssm_state, void* conv_state, void* y,
                             int64_t n_layers, int64_t batch, int64_t d_inner,
                             int64_t d_state, int64_t d_conv, mm_dtype act, void* stream)
{
    if (act != MM_F32 && act != MM_BF16) return MM_ERR_DTYPE;
    if (n_layers < 0 || batch < 0 || d_inner <= 0 || d_state <= 0 || d_conv <= 0) return MM_ERR_SHAPE;
    if (d_state != 16 || d_conv != 4 || d_inner % 8 != 0) return MM_ERR_UNSUPPORTED;
    if (d_inner > (1 << 24) || batch > (1 << 24) || n_layers > (1 << 24)) return MM_ERR_SHAPE;
    const int64_t es = act == MM_F32 ? 4 : 2;
    int64_t lb, rows, st_bytes;
    if (!mul_ok(n_layers, batch, &lb) || !mul_ok(lb, d_inner, &rows) || !mul_ok(rows, d_state * 4, &st_bytes))
        return MM_ERR_SHAPE;
    if (rows == 0) return MM_OK;
    // one warp per (layer, 32-channel block, chunk of batch rows); warps <= rows
    const int64_t warps = n_layers * ((d_inner + 31) / 32) *
                          ((batch + mm::kDecodeBatchChunk - 1) / mm::kDecodeBatchChunk);
    if ((warps + 7) / 8 > INT32_MAX) return MM_ERR_SHAPE;

    if (!x || !z || !dt || !conv_w || !dt_bias || !A || !Bm || !Cm || !ssm_state || !conv_state || !y)
        return MM_ERR_NULL;
    const void* all[] = {x, z, dt, conv_w, conv_b, dt_bias, Dskip, A, Bm, Cm, ssm_state, conv_state, y};
    for (const void* q : all)
        if (q && !aligned16(q)) return MM_ERR_ALIGN;

    const int64_t tok_bytes = rows * es;
    const int64_t par = n_layers * d_inner * 4;
    const Span in[] = {span(x, tok_bytes), span(z, tok_bytes), span(dt, tok_bytes),
                       span(conv_w, par * d_conv), span(conv_b, par), span(dt_bias, par), span(Dskip, par),
                       span(A, par * d_state), span(Bm, lb * d_state * es), span(Cm, lb * d_state * es)};
    const Span io[] = {span(ssm_state, st_bytes), span(conv_state, rows * (d_conv - 1) * es), span(y, tok_bytes)};
    for (const Span& o : io)
        for (const Span& i : in)
            if (overlaps(o, i)) return MM_ERR_ALIAS;
    if (overlaps(io[0], io[1]) || overlaps(io[0], io[2]) || overlaps(io[1], io[2])) return MM_ERR_ALIAS;

    int sm_count = 0;
    if (mm_status st = check_device(&sm_count); st != MM_OK) return st;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const unsigned grid = static_cast<unsigned>((warps + 7) / 8);
    if (act == MM_BF16) {
        using T = __nv_bfloat16;
        mm::state_update_kernel<T, mm::MathFast><<<grid, 256, 0, s>>>(
            static_cast<const T*>(x), static_cast<const T*>(z), static_cast<const T*>(dt), conv_w, conv_b,
            dt_bias, Dskip, A, static_cast<const T*>(Bm), static_cast<const T*>(Cm), ssm_state,
            static_cast<T*>(conv_state), static_cast<T*>(y), static_cast<int>(n_layers), static_cast<int>(batch),
            static_cast<int>(d_inner));
    } else {
        mm::state_update_kernel<float, mm::MathExact><<<grid, 256, 0, s>>>(
            static_cast<const float*>(x), static_cast<const float*>(z), static_cast<const float*>(dt), conv_w,
            conv_b, dt_bias, Dskip, A, static_cast<const float*>(Bm), static_cast<const float*>(Cm), ssm_state,
            static_cast<float*>(conv_state), static_cast<float*>(y), static_cast<int>(n_layers),
            static_cast<int>(batch), static_cast<int>(d_inner));
    }
    if (cudaGetLastError() != cudaSuccess) return MM_ERR_CUDA;
    return MM_OK;
}

mm_status mamba_mixer_fwd_noalloc(const void* xz, const float* conv_w, const float* conv_b,
                                  const void* dt, const float* dt_bias, const float* A,
                                  const void* Bm, const void* Cm, const float* Dskip,
                                  const float* h0, const void* conv_state_in,
                                  void* y, float* h_last, void* conv_state_out,
                                  int64_t batch, int64_t seqlen, int64_t d_inner,
                                  int64_t d_state, int64_t d_conv, mm_dtype act, void* stream)
{
    const size_t need = mamba_mixer_workspace_size(batch, seqlen, d_inner, d_state, d_conv, act);
    if (need > MAMBA_MIXER_NOALLOC_SCRATCH_BYTES) return MM_ERR_SCRATCH_LIMIT;
    void* scratch = nullptr;
    if (need > 0) {
        if (mm_status st = noalloc_scratch(&scratch); st != MM_OK) return st;
    }
    return mamba_mixer_fwd(xz, conv_w, conv_b, dt, dt_bias, A, Bm, Cm, Dskip, h0, conv_state_in, y, h_last,
                           conv_state_out, batch, seqlen, d_inner, d_state, d_conv, act, scratch,
                           need > 0 ? MAMBA_MIXER_NOALLOC_SCRATCH_BYTES : 0, stream);
}

size_t mamba_mixer_host_workspace_size(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state,
                                       int64_t d_conv, mm_dtype act) {
    if ((act != MM_F32 && act != MM_BF16) || batch <= 0 || seqlen < 0 || d_inner <= 0 || d_state != 16 ||
        d_conv != 4 || d_inner % 8 != 0 || d_inner > (1 << 24) || batch > (1 << 24))
        return 0;
    int64_t tokens, bytes;
    if (!mul_ok(batch, seqlen, &tokens) || !mul_ok(tokens, 2 * d_inner * 4, &bytes)) return 0;
    const int64_t es = act == MM_F32 ? 4 : 2;
    const HostPlan hp = plan_host(batch, seqlen, d_inner, es);
    return seqlen_ok(hp.piece, d_inner, es) ? hp.total : 0;
}

mm_status mamba_mixer_fwd_host(const void* xz, const float* conv_w, const float* conv_b,
                               const void* dt, const float* dt_bias, const float* A,
                               const void* Bm, const void* Cm, const float* Dskip,
                               const float* h0, const void* conv_state_in,
                               void* y, float* h_last, void* conv_state_out,
                               int64_t batch, int64_t seqlen, int64_t d_inner,
                               int64_t d_state, int64_t d_conv, mm_dtype act,
                               void* workspace, size_t workspace_bytes,
                               void* stream, void* h2d_stream, void* d2h_stream)
{
    if (act != MM_F32 && act != MM_BF16) return MM_ERR_DTYPE;
    if (batch < 0 || seqlen < 0 || d_inner <= 0 || d_state <= 0 || d_conv <= 0) return MM_ERR_SHAPE;
    if (d_state != 16 || d_conv != 4 || d_inner % 8 != 0) return MM_ERR_UNSUPPORTED;
    if (d_inner > (1 << 24) || batch > (1 << 24)) return MM_ERR_SHAPE;
    const int64_t es = act == MM_F32 ? 4 : 2;
    int64_t tokens, xz_bytes, dt_bytes, bc_bytes, st_bytes;
    if (!mul_ok(batch, seqlen, &tokens) || !mul_ok(tokens, 2 * d_inner * es, &xz_bytes) ||
        !mul_ok(tokens, d_inner * es, &dt_bytes) || !mul_ok(tokens, d_state * es, &bc_bytes) ||
        !mul_ok(batch, d_inner * d_state * 4, &st_bytes))
        return MM_ERR_SHAPE;
    const int64_t cs_bytes = batch * d_inner * (d_conv - 1) * es;
    if (batch == 0) return MM_OK;

    if (!conv_w || !dt_bias || !A || !h_last || !conv_state_out) return MM_ERR_NULL;
    if (seqlen > 0 && (!xz || !dt || !Bm || !Cm || !y)) return MM_ERR_NULL;
    // device pointers and the workspace: 16-byte aligned (host buffers need not be)
    const void* dev_ptrs[] = {conv_w, conv_b, dt_bias, A, Dskip};
    for (const void* q : dev_ptrs)
        if (q && !aligned16(q)) return MM_ERR_ALIGN;
    // host outputs may not overlap host inputs
    const Span in[] = {span(xz, xz_bytes), span(dt, dt_bytes), span(Bm, bc_bytes), span(Cm, bc_bytes),
                       span(h0, st_bytes), span(conv_state_in, cs_bytes)};
    const Span out[] = {span(y, dt_bytes), span(h_last, st_bytes), span(conv_state_out, cs_bytes)};
    for (const Span& o : out)
        for (const Span& i : in)
            if (overlaps(o, i)) return MM_ERR_ALIAS;
    if (overlaps(out[0], out[1]) || overlaps(out[0], out[2]) || overlaps(out[1], out[2])) return MM_ERR_ALIAS;

    const HostPlan hp = plan_host(batch, seqlen, d_inner, es);
    if (!seqlen_ok(hp.piece, d_inner, es)) return MM_ERR_SHAPE;   // each piece is one device call
    if (!workspace || workspace_bytes < hp.total) return MM_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MM_ERR_ALIGN;
    int sm_count = 0;
    if (mm_status st = check_device(&sm_count); st != MM_OK) return st;

    cudaStream_t sc = static_cast<cudaStream_t>(stream);
    cudaStream_t s_in = static_cast<cudaStream_t>(h2d_stream);
    cudaStream_t s_out = static_cast<cudaStream_t>(d2h_stream);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    unsigned char* slot[2] = {ws, ws + hp.slot};
    unsigned char* carry[2] = {ws + 2 * hp.slot, ws + 2 * hp.slot + hp.carry};
    void* fwd_ws = hp.fwd_ws ? ws + 2 * hp.slot + 2 * hp.carry : nullptr;

    HostEvents evs;
    cudaEvent_t ev_start = evs.make(), ev_final = evs.make();
    cudaEvent_t ev_in[2] = {evs.make(), evs.make()};
    cudaEvent_t ev_done[2] = {evs.make(), evs.make()};
    cudaEvent_t ev_free[2] = {evs.make(), evs.make()};
    if (evs.n != 8) { cudaGetLastError(); return MM_ERR_CUDA; }

    bool ok = true;
    mm_status fwd_status = MM_OK;
    auto chk = [&](cudaError_t e) { ok = ok && e == cudaSuccess; };
    const size_t B = static_cast<size_t>(batch), D = static_cast<size_t>(d_inner), e = static_cast<size_t>(es);
    const size_t L = static_cast<size_t>(seqlen);
    const unsigned char* xz_h = static_cast<const unsigned char*>(xz);
    const unsigned char* dt_h = static_cast<const unsigned char*>(dt);
    const unsigned char* b_h = static_cast<const unsigned char*>(Bm);
    const unsigned char* c_h = static_cast<const unsigned char*>(Cm);
    unsigned char* y_h = static_cast<unsigned char*>(y);

    // the copies touch the workspace, which the caller's earlier work on `stream` may still use
    chk(cudaEventRecord(ev_start, sc));
    chk(cudaStreamWaitEvent(s_in, ev_start, 0));
    chk(cudaStreamWaitEvent(s_out, ev_start, 0));
    if (h0) chk(cudaMemcpyAsync(carry[0], h0, static_cast<size_t>(st_bytes), cudaMemcpyHostToDevice, s_in));
    if (conv_state_in)
        chk(cudaMemcpyAsync(carry[0] + hp.carry_h, conv_state_in, static_cast<size_t>(cs_bytes),
                            cudaMemcpyHostToDevice, s_in));

    for (int64_t i = 0; ok && i < hp.pieces; ++i) {
        const int j = static_cast<int>(i & 1);
        int64_t pt0 = 0, pn = 0;
        piece_range(hp, i, seqlen, &pt0, &pn);
        const size_t t0 = static_cast<size_t>(pt0), n = static_cast<size_t>(pn);
        unsigned char* sl = slot[j];
        // inputs of piece i -> slot j, once the piece that used the slot has been copied out
        if (i >= 2) chk(cudaStreamWaitEvent(s_in, ev_free[j], 0));
        if (n > 0) {
            chk(cudaMemcpy2DAsync(sl, n * 2 * D * e, xz_h + t0 * 2 * D * e, L * 2 * D * e, n * 2 * D * e, B,
                                  cudaMemcpyHostToDevice, s_in));
            chk(cudaMemcpy2DAsync(sl + hp.off_dt, n * D * e, dt_h + t0 * D * e, L * D * e, n * D * e, B,
                                  cudaMemcpyHostToDevice, s_in));
            chk(cudaMemcpy2DAsync(sl + hp.off_b, n * 16 * e, b_h + t0 * 16 * e, L * 16 * e, n * 16 * e, B,
                                  cudaMemcpyHostToDevice, s_in));
            chk(cudaMemcpy2DAsync(sl + hp.off_c, n * 16 * e, c_h + t0 * 16 * e, L * 16 * e, n * 16 * e, B,
                                  cudaMemcpyHostToDevice, s_in));
        }
        chk(cudaEventRecord(ev_in[j], s_in));
        // the forward of piece i, carrying the state from piece i-1
        chk(cudaStreamWaitEvent(sc, ev_in[j], 0));
        unsigned char* cin = carry[i & 1];
        unsigned char* cout = carry[(i + 1) & 1];
        const bool first = i == 0;
        const float* h_in = (first && !h0) ? nullptr : reinterpret_cast<const float*>(cin);
        const void* cs_in = (first && !conv_state_in) ? nullptr : cin + hp.carry_h;
        if (!ok) break;
        fwd_status = mamba_mixer_fwd(sl, conv_w, conv_b, sl + hp.off_dt, dt_bias, A, sl + hp.off_b,
                                             sl + hp.off_c, Dskip, h_in, cs_in, sl + hp.off_y,
                                             reinterpret_cast<float*>(cout), cout + hp.carry_h, batch,
                                             static_cast<int64_t>(n), d_inner, d_state, d_conv, act, fwd_ws,
                                             hp.fwd_ws, sc);
        if (fwd_status != MM_OK) break;
        chk(cudaEventRecord(ev_done[j], sc));
        // y of piece i -> host; the slot is free again after this copy
        chk(cudaStreamWaitEvent(s_out, ev_done[j], 0));
        if (n > 0)
            chk(cudaMemcpy2DAsync(y_h + t0 * D * e, L * D * e, sl + hp.off_y, n * D * e, n * D * e, B,
                                  cudaMemcpyDeviceToHost, s_out));
        chk(cudaEventRecord(ev_free[j], s_out));
    }
    // the carried state after the last piece -> host; `stream` then waits for every
    // copy queued so far (also after a failure, so the caller can sync `stream`
    // before releasing its buffers)
    if (ok && fwd_status == MM_OK) {
        unsigned char* cl = carry[hp.pieces & 1];
        chk(cudaMemcpyAsync(h_last, cl, static_cast<size_t>(st_bytes), cudaMemcpyDeviceToHost, s_out));
        chk(cudaMemcpyAsync(conv_state_out, cl + hp.carry_h, static_cast<size_t>(cs_bytes),
                            cudaMemcpyDeviceToHost, s_out));
    }
    const bool fenced = cudaEventRecord(ev_final, s_out) == cudaSuccess &&
                        cudaEventRecord(ev_in[0], s_in) == cudaSuccess &&
                        cudaStreamWaitEvent(sc, ev_final, 0) == cudaSuccess &&
                        cudaStreamWaitEvent(sc, ev_in[0], 0) == cudaSuccess;
    if (fwd_status != MM_OK) return fwd_status;
    if (!ok || !fenced) { cudaGetLastError(); return MM_ERR_CUDA; }
    return MM_OK;
}

}  // extern "C"
