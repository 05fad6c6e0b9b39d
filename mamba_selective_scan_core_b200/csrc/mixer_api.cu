// Host side of the C ABI declared in include/mamba_mixer.h: argument
// validation (before anything is launched), launch-plan and CTA-shape
// selection, and the launches themselves.  No allocation.  The library's
// state is the device fault word, the fixed scratch array of
// mamba_mixer_fwd_noalloc with its per-context address, a call counter, and
// host-side caches (SM counts, kernel attributes already set, recent tensor
// maps) that only save repeated work.
#include <algorithm>
#include <atomic>
#include <cudaTypedefs.h>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "mamba_mixer.h"
#include "mixer_decode.cuh"
#include "mixer_prefill.cuh"
#include "proj_gemm.cuh"
#include "proj_ops.cuh"
#include "ssd.cuh"
#include "m3.cuh"

namespace {

using mm::PrefillLayout;
using mm::PrefillParams;

constexpr int kTile = 32;
constexpr int kMaxThreads = 128;
constexpr int kSmemBudget = 200 * 1024;
constexpr int kMaxDevices = 256;

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

int env_int(const char* name, int lo, int hi) {
    if (const char* e = std::getenv(name)) {
        const int v = std::atoi(e);
        if (v >= lo && v <= hi) return v;
    }
    return 0;
}

// ---------------------------------------------------------------- devices
// SM count of the current device, queried once per device.  Without a usable
// device the plan falls back to a B200's 148 SMs, so that sizes computed on a
// machine without a GPU describe the B200 plan.
constexpr int kB200SMs = 148;

int plan_sms() {
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return kB200SMs;
    }
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return kB200SMs;
    }
    cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// The current device must be an sm_100 part (B200).
mm_status check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return MM_ERR_DEVICE; }
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
        cudaGetLastError();
        return MM_ERR_DEVICE;
    }
    return major == 10 ? MM_OK : MM_ERR_DEVICE;
}

// Ids of launch pairs and per-call status epochs: unique in the process,
// never 0, below 2^56 (the status word keeps 8 bits for the code).
std::atomic<unsigned long long> g_call_counter{0};
unsigned long long next_call_id() { return (g_call_counter.fetch_add(1) + 1) & ((1ull << 56) - 1); }

// ---------------------------------------------------------------- launch plan
// Launch plan of a forward call: time chunks, and the workspace they need.
// A function of the sizes, the current device's SM count and the
// MAMBA_MIXER_CHUNKS tuning variable, so that mamba_mixer_workspace_size()
// and the call agree.
//
// Workspace layout (every region 256-byte aligned):
//   header  [256 B]                   the call status (PrefillParams::ws_hdr)
//   tags    [K-1][batch][D/8] u64     who wrote each summary (PrefillParams::ws_tags)
//   state   [K-1][batch][16][D] f32   chunk end states from zero
//   lsum    [K-1][batch][D] f32       chunk step-size sums
struct FwdPlan {
    int chunks = 1;
    int64_t chunk0_len = 0;   // tokens of chunk 0
    int64_t chunk_len = 0;    // tokens of every later chunk (the last one may be shorter)
    size_t off_tags = 0, off_state = 0, off_lsum = 0, ws_bytes = 0;
};

constexpr size_t kWsHeader = 256;
constexpr int kMinBlocksFwd = MM_FWD_MIN_BLOCKS;
constexpr int kWarpsPerSM = 4 * kMinBlocksFwd;   // resident warps per SM at the forward's register use
constexpr int kMinChunkTiles = 4;        // shortest chunk worth a summary pass
constexpr int kMaxChunks = 16;

size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

// Tries per wait on a bulk copy (each try waits a bounded time in hardware):
// about a second by default; MAMBA_MIXER_WAIT_LIMIT overrides it (tests use 0
// to make the wait give up at once).
// MAMBA_MIXER_SUMMARY_WAIT_LIMIT applies to the summary pass alone (tests use
// it to make only the summaries go missing).
unsigned env_wait_limit(const char* name, unsigned dflt) {
    if (const char* e = std::getenv(name)) {
        char* end = nullptr;
        const long v = std::strtol(e, &end, 10);
        if (end != e && v >= 0 && v <= (1L << 30)) return static_cast<unsigned>(v);
    }
    return dflt;
}
unsigned copy_wait_limit() { return env_wait_limit("MAMBA_MIXER_WAIT_LIMIT", 1u << 20); }

// Time chunks.  More chunks put more warps on the SMs but add a summary pass
// over (K-1)/K of the tokens, so K minimises a measured cost model: a pass
// takes about (tokens per chunk) x (time of its busiest SM), an SM running
// 8 warps (two CTAs) taking ~1.85x as long as one running 4, and a summary
// token costing ~0.55 of a full-pass token (B200 measurements of both
// kernels), among splits that fit one wave.  It picks 9 chunks for one
// 8192-channel sequence on 148 SMs and a single chunk once a batch fills the
// SMs on its own.
double busiest_sm(int64_t warps, int sms) {
    const int64_t m = (warps + sms - 1) / sms;        // warps on the busiest SM
    const int64_t waves = m / kWarpsPerSM, rest = m % kWarpsPerSM;
    return 1.85 * static_cast<double>(waves) + (rest == 0 ? 0.0 : rest * 2 <= kWarpsPerSM ? 1.0 : 1.85);
}

FwdPlan plan_fwd(int64_t batch, int64_t seqlen, int64_t d_inner, int sms) {
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
            if (chunks > 1 && chunks * warps > static_cast<int64_t>(sms) * kWarpsPerSM) break;
            const double cost = static_cast<double>(ct) *
                                (busiest_sm(chunks * warps, sms) +
                                 (chunks > 1 ? 0.55 * busiest_sm((chunks - 1) * warps, sms) : 0.0));
            if (c == 1 || cost < best) { best = cost; k = c; }
        }
    }
    pl.chunk_len = chunk_tiles(k) * kTile;
    pl.chunk0_len = pl.chunk_len;
    pl.chunks = static_cast<int>(seqlen > 0 ? (seqlen + pl.chunk_len - 1) / pl.chunk_len : 1);
    // Chunk 0 needs no carried state, so its full pass runs while the summary
    // pass runs; chunks 1.. start once every summary is stored.  The call then
    // takes about max(l0, (1 + 0.55) l1) in tile units, with l0 the tiles of
    // chunk 0 and l1 those of every other chunk: a longer chunk 0 and even
    // chunks after it (instead of equal chunks and a short last one).
    if (pl.chunks > 1 && !env_int("MAMBA_MIXER_CHUNKS", 1, 1 << 20)) {
        const int64_t K = pl.chunks;
        double best = 1e300;
        int64_t best_l1 = 0;
        for (int64_t l1 = 1; l1 * (K - 1) < tiles; ++l1) {
            const int64_t l0 = tiles - l1 * (K - 1);
            const double t = std::max(static_cast<double>(l0), 1.55 * static_cast<double>(l1));
            if (t < best) { best = t; best_l1 = l1; }
        }
        if (best_l1 > 0) {
            pl.chunk_len = best_l1 * kTile;
            pl.chunk0_len = (tiles - best_l1 * (K - 1)) * kTile;
        }
    }
    const size_t c1 = static_cast<size_t>(pl.chunks - 1), B = static_cast<size_t>(batch);
    const size_t D = static_cast<size_t>(d_inner);
    pl.off_tags = kWsHeader;
    pl.off_state = pl.off_tags + align256(c1 * B * (D / 8) * sizeof(unsigned long long));
    pl.off_lsum = pl.off_state + align256(c1 * B * 16 * D * sizeof(float));
    pl.ws_bytes = pl.off_lsum + align256(c1 * B * D * sizeof(float));
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

// A map is a pure function of its base address, sizes and box; each host
// thread keeps its most recent ones, so repeated calls on the same buffers
// (a serving loop, a benchmark) skip the encoder.
struct MapKey {
    const void* base;
    int64_t cols, rows, batch;
    int box_cols, box_rows;
    bool bf16;
    bool operator==(const MapKey& o) const {
        return base == o.base && cols == o.cols && rows == o.rows && batch == o.batch && box_cols == o.box_cols &&
               box_rows == o.box_rows && bf16 == o.bf16;
    }
};
constexpr int kMapCache = 20;
struct MapCache {
    MapKey key[kMapCache];
    CUtensorMap map[kMapCache];
    int n = 0, next = 0;
};
thread_local MapCache t_maps;

// 3-D map over a [batch][rows][cols] tensor with a [1][box_rows][box_cols] box.
bool encode_3d(CUtensorMap* m, const void* base, bool bf16, int64_t cols, int64_t rows, int64_t batch,
               int box_cols, int box_rows) {
    const MapKey k{base, cols, rows, batch, box_cols, box_rows, bf16};
    MapCache& c = t_maps;
    for (int i = 0; i < c.n; ++i)
        if (c.key[i] == k) { *m = c.map[i]; return true; }
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const int64_t es = bf16 ? 2 : 4;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                                static_cast<cuuint64_t>(batch)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols * es), static_cast<cuuint64_t>(rows * cols * es)};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    const int slot = c.n < kMapCache ? c.n++ : c.next;
    c.next = (slot + 1) % kMapCache;
    c.key[slot] = k;
    c.map[slot] = *m;
    return true;
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

// Every launch asks for at most kSmemBudget bytes of dynamic shared memory
// (ring_depth guarantees it); each kernel is allowed that much once per device
// (the attribute belongs to the kernel in that device's context).  `done` is
// the per-kernel record of devices already set.
template <typename Kern>
cudaError_t allow_smem(Kern kern, std::atomic<unsigned long long>& done) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaGetLastError();
    const unsigned long long bit = dev < 64 ? 1ull << dev : 0;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// Test hook: MAMBA_MIXER_TEST_LAUNCH_FAIL=1 makes every forward launch ask
// for more dynamic shared memory than any CTA may have, so the runtime
// rejects it on the host (nothing reaches the GPU) and the call returns
// MM_ERR_CUDA; the next call without it runs normally.
bool forced_launch_failure() { return env_int("MAMBA_MIXER_TEST_LAUNCH_FAIL", 1, 1) == 1; }

// `dependent`: launch as a programmatic dependent of the kernel before it in
// the stream (the summary pass of the same call), see mixer_fwd_kernel.
template <typename T, typename M, int STAGES, bool SUMMARY, int OCT = 0>
cudaError_t launch_prefill(const PrefillParams& p, int64_t batch, int chunks, int threads, bool dependent,
                           cudaStream_t s) {
    auto kern = mm::mixer_fwd_kernel<T, M, kTile, STAGES, SUMMARY, OCT>;
    TensorMaps maps;
    if (!make_maps<T>(p, batch, &maps)) return cudaErrorInvalidValue;
    const int smem = PrefillLayout<T>::smem_bytes(kTile, STAGES, p.octets);
    static std::atomic<unsigned long long> smem_allowed{0};   // one record per kernel instance
    cudaError_t e = allow_smem(kern, smem_allowed);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(batch * p.ctas_per_seq), static_cast<unsigned>(chunks));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = forced_launch_failure() ? size_t(1) << 20 : static_cast<size_t>(smem);
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

struct CtaShape {
    int octets = 1, ctas_per_seq = 1, threads = 32, stages = 2;
};

template <typename T>
CtaShape shape_ctas(int64_t d_inner, int64_t batch, int64_t chunks, int sm_count) {
    const int64_t octets_per_seq = d_inner / 8;
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
    CtaShape sh;
    const int64_t ctas = (octets_per_seq + best - 1) / best;
    sh.octets = static_cast<int>((octets_per_seq + ctas - 1) / ctas);
    sh.ctas_per_seq = static_cast<int>(ctas);
    sh.threads = ((sh.octets * 4) + 31) / 32 * 32;
    sh.stages = std::min(best_stages, std::max(2, ring_depth<T>(sh.octets)));
    return sh;
}

template <typename T, typename M, bool SUMMARY>
cudaError_t launch_pass(PrefillParams p, const CtaShape& sh, int64_t batch, int chunks, bool dependent,
                        cudaStream_t s) {
    p.octets = sh.octets;
    p.ctas_per_seq = sh.ctas_per_seq;
    // the widest CTA (256 channels) of the bf16 path, the shape of wide layers,
    // with its row width as a compile-time constant
    if constexpr (std::is_same<T, __nv_bfloat16>::value && std::is_same<M, mm::MathFast>::value) {
        if (sh.octets == 32 && sh.stages == 2 && env_int("MAMBA_MIXER_GENERIC_WIDTH", 1, 1) == 0)
            return launch_prefill<T, M, 2, SUMMARY, 32>(p, batch, chunks, sh.threads, dependent, s);
    }
    if (sh.stages >= 4) return launch_prefill<T, M, 4, SUMMARY>(p, batch, chunks, sh.threads, dependent, s);
    if (sh.stages == 3) return launch_prefill<T, M, 3, SUMMARY>(p, batch, chunks, sh.threads, dependent, s);
    return launch_prefill<T, M, 2, SUMMARY>(p, batch, chunks, sh.threads, dependent, s);
}

template <typename T, typename M>
cudaError_t dispatch_prefill(PrefillParams p, int64_t batch, const FwdPlan& pl, int sm_count, cudaStream_t s) {
    p.chunk_len = pl.chunk_len;
    p.chunk0_len = pl.chunk0_len;
    p.n_chunks = pl.chunks;
    // checked build's test hook: MAMBA_MIXER_TEST_BOUNDS_SHRINK=k takes k
    // elements off the extent the kernels check y's stores against (the buffer
    // itself is whole): the last k elements' stores are skipped and reported
    p.check_shrink = mm::kCheckBounds ? env_int("MAMBA_MIXER_TEST_BOUNDS_SHRINK", 1, 1 << 30) : 0;
    // the summary pass takes every token of its chunks as valid: they must be
    // whole tiles that end inside the sequence
    if (pl.chunks > 1 && (pl.chunk0_len % kTile != 0 || pl.chunk_len % kTile != 0 ||
                          pl.chunk0_len + static_cast<int64_t>(pl.chunks - 2) * pl.chunk_len > p.L))
        return cudaErrorInvalidValue;
    const CtaShape full = shape_ctas<T>(p.D, batch, pl.chunks, sm_count);
    // The summary pass is launched normally: it starts after everything
    // before it in the stream, the producers of the inputs included.  The
    // full pass follows it as a programmatic dependent; its CTAs read the
    // inputs freely (they were complete before the summary pass started) and
    // wait for the summary grid before reading its results.
    if (pl.chunks > 1) {
        const CtaShape sum = shape_ctas<T>(p.D, batch, pl.chunks - 1, sm_count);
        p.sum_octets = sum.octets;
        PrefillParams ps = p;
        ps.wait_limit = env_wait_limit("MAMBA_MIXER_SUMMARY_WAIT_LIMIT", p.wait_limit);
        cudaError_t e = launch_pass<T, M, true>(ps, sum, batch, pl.chunks - 1, false, s);
        if (e != cudaSuccess) return e;
    }
    return launch_pass<T, M, false>(p, full, batch, pl.chunks, pl.chunks > 1, s);
}

// ---------------------------------------------------------------- forward calls
// The arguments of a forward call, as the entry points receive them.
struct FwdArgs {
    const void* xz; const float* conv_w; const float* conv_b; const void* dt; const float* dt_bias;
    const float* A; const void* Bm; const void* Cm; const float* Dskip; const float* h0;
    const void* cs_in; void* y; float* h_last; void* cs_out;
    int64_t batch, seqlen, d_inner, d_state, d_conv;
    mm_dtype act;
    const float* b_norm_w = nullptr;   // optional RMSNorm of B_t / C_t ([d_state] each)
    const float* c_norm_w = nullptr;
    float norm_eps = 0.0f;
};

struct FwdBytes {
    int64_t es = 0, xz = 0, dt = 0, bc = 0, st = 0, cs = 0;
};

// Sizes and dtype: the checks shared by every forward entry point.
mm_status check_sizes(const FwdArgs& a, FwdBytes* nb) {
    if (a.act != MM_F32 && a.act != MM_BF16) return MM_ERR_DTYPE;
    if (a.batch < 0 || a.seqlen < 0 || a.d_inner <= 0 || a.d_state <= 0 || a.d_conv <= 0) return MM_ERR_SHAPE;
    if (a.d_state != 16 || a.d_conv != 4 || a.d_inner % 8 != 0) return MM_ERR_UNSUPPORTED;
    if (a.d_inner > (1 << 24) || a.batch > (1 << 24)) return MM_ERR_SHAPE;
    nb->es = a.act == MM_F32 ? 4 : 2;
    int64_t tokens;
    if (!mul_ok(a.batch, a.seqlen, &tokens) || !mul_ok(tokens, 2 * a.d_inner * nb->es, &nb->xz) ||
        !mul_ok(tokens, a.d_inner * nb->es, &nb->dt) || !mul_ok(tokens, a.d_state * nb->es, &nb->bc) ||
        !mul_ok(a.batch, a.d_inner * a.d_state * 4, &nb->st))
        return MM_ERR_SHAPE;
    nb->cs = a.batch * a.d_inner * (a.d_conv - 1) * nb->es;
    return MM_OK;
}

// Every check of a device-memory forward call except the workspace.
mm_status validate_fwd(const FwdArgs& a, FwdBytes* nb) {
    if (mm_status st = check_sizes(a, nb); st != MM_OK) return st;
    if (!seqlen_ok(a.seqlen, a.d_inner, nb->es)) return MM_ERR_SHAPE;
    if (a.batch == 0) return MM_OK;
    if (!a.conv_w || !a.dt_bias || !a.A || !a.h_last || !a.cs_out) return MM_ERR_NULL;
    if (a.seqlen > 0 && (!a.xz || !a.dt || !a.Bm || !a.Cm || !a.y)) return MM_ERR_NULL;
    if ((a.b_norm_w || a.c_norm_w) && !(a.norm_eps > 0.0f && a.norm_eps < 1e30f)) return MM_ERR_ARG;
    const void* all[] = {a.xz, a.conv_w, a.conv_b, a.dt, a.dt_bias, a.A, a.Bm, a.Cm, a.Dskip, a.h0, a.cs_in,
                         a.y, a.h_last, a.cs_out, a.b_norm_w, a.c_norm_w};
    for (const void* q : all)
        if (q && !aligned16(q)) return MM_ERR_ALIGN;
    const int64_t D = a.d_inner;
    const Span in[] = {span(a.xz, nb->xz), span(a.conv_w, D * a.d_conv * 4), span(a.conv_b, D * 4),
                       span(a.dt, nb->dt), span(a.dt_bias, D * 4), span(a.A, D * a.d_state * 4),
                       span(a.Bm, nb->bc), span(a.Cm, nb->bc), span(a.Dskip, D * 4),
                       span(a.h0, nb->st), span(a.cs_in, nb->cs), span(a.b_norm_w, a.d_state * 4),
                       span(a.c_norm_w, a.d_state * 4)};
    const Span out[] = {span(a.y, nb->dt), span(a.h_last, nb->st), span(a.cs_out, nb->cs)};
    for (const Span& o : out)
        for (const Span& i : in)
            if (overlaps(o, i)) return MM_ERR_ALIAS;
    if (overlaps(out[0], out[1]) || overlaps(out[0], out[2]) || overlaps(out[1], out[2])) return MM_ERR_ALIAS;
    return MM_OK;
}

// The workspace (or scratch) may overlap no input or output.
bool workspace_overlaps(const FwdArgs& a, const FwdBytes& nb, const void* ws, size_t bytes) {
    const int64_t D = a.d_inner;
    const Span w = span(ws, static_cast<int64_t>(bytes));
    const Span all[] = {span(a.xz, nb.xz), span(a.conv_w, D * a.d_conv * 4), span(a.conv_b, D * 4),
                        span(a.dt, nb.dt), span(a.dt_bias, D * 4), span(a.A, D * a.d_state * 4),
                        span(a.Bm, nb.bc), span(a.Cm, nb.bc), span(a.Dskip, D * 4), span(a.h0, nb.st),
                        span(a.cs_in, nb.cs), span(a.y, nb.dt), span(a.h_last, nb.st), span(a.cs_out, nb.cs),
                        span(a.b_norm_w, a.d_state * 4), span(a.c_norm_w, a.d_state * 4)};
    for (const Span& s : all)
        if (overlaps(w, s)) return true;
    return false;
}

// Launch a validated forward (batch > 0) on `ws`, laid out as `pl` says.
// Its failures are recorded in ws's header under `status_epoch`.
mm_status run_fwd(const FwdArgs& a, const FwdPlan& pl, int sm_count, void* ws, unsigned long long status_epoch,
                  cudaStream_t s) {
    unsigned char* w = static_cast<unsigned char*>(ws);
    PrefillParams p{};
    p.xz = a.xz; p.conv_w = a.conv_w; p.conv_b = a.conv_b; p.dt = a.dt; p.dt_bias = a.dt_bias; p.A = a.A;
    p.Bm = a.Bm; p.Cm = a.Cm; p.Dskip = a.Dskip; p.h0 = a.h0; p.cs_in = a.cs_in;
    p.y = a.y; p.h_last = a.h_last; p.cs_out = a.cs_out;
    p.L = a.seqlen;
    p.D = static_cast<int>(a.d_inner);
    p.batch = static_cast<int>(a.batch);
    p.wait_limit = copy_wait_limit();
    p.ws_hdr = reinterpret_cast<unsigned long long*>(w);
    p.ws_tags = reinterpret_cast<unsigned long long*>(w + pl.off_tags);
    p.ws_state = reinterpret_cast<float*>(w + pl.off_state);
    p.ws_lsum = reinterpret_cast<float*>(w + pl.off_lsum);
    p.call_id = next_call_id();
    p.status_epoch = status_epoch;
    p.sum_octets = 1;
    p.b_norm_w = a.b_norm_w;
    p.c_norm_w = a.c_norm_w;
    p.norm_eps = a.norm_eps;
    cudaError_t e = a.act == MM_BF16 ? dispatch_prefill<__nv_bfloat16, mm::MathFast>(p, a.batch, pl, sm_count, s)
                                     : dispatch_prefill<float, mm::MathExact>(p, a.batch, pl, sm_count, s);
    if (e != cudaSuccess) { cudaGetLastError(); return MM_ERR_CUDA; }
    return MM_OK;
}

// ---------------------------------------------------------------- host-memory forward
// Piece plan of mamba_mixer_fwd_host: the sequence is cut into about
// kHostPieces pieces (whole tiles, at least kHostMinPiece tokens) and the
// device workspace holds the piece forward's own workspace first (so that
// mamba_check_status reads the call's status from the workspace's start),
// then two staging slots and two carried states (ping-pong), each region
// 256-byte aligned.  What follows the last input copy -- the last piece's
// forward and the copy back of its y -- is the call's tail, so a last piece of
// at least kHostMinPiece tokens is cut once more, in two.
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

// First token and length of piece i of a plan over `seqlen` tokens.
void piece_range(const HostPlan& hp, int64_t i, int64_t seqlen, int64_t* t0, int64_t* n) {
    const int64_t tail = hp.head * hp.piece;
    if (i < hp.head) { *t0 = i * hp.piece; *n = hp.piece; }
    else if (hp.tail1 == 0) { *t0 = tail; *n = seqlen - tail; }
    else if (i == hp.head) { *t0 = tail; *n = hp.tail1; }
    else { *t0 = tail + hp.tail1; *n = seqlen - tail - hp.tail1; }
}

HostPlan plan_host(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t es, int sms) {
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
    // the piece workspace must fit the plan of every piece length used
    size_t ws = plan_fwd(batch, hp.tail1 > 0 ? hp.tail1 : rest, d_inner, sms).ws_bytes;
    if (hp.head > 0) ws = std::max(ws, plan_fwd(batch, hp.piece, d_inner, sms).ws_bytes);
    if (hp.tail1 > 0) ws = std::max(ws, plan_fwd(batch, rest - hp.tail1, d_inner, sms).ws_bytes);
    hp.fwd_ws = align256(ws);
    hp.total = hp.fwd_ws + 2 * hp.slot + 2 * hp.carry;
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
// ever passes its device address (looked up per context, below) to kernels.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MAMBA_MIXER_NOALLOC_SCRATCH_BYTES];

namespace {

// The driver's context queries, fetched through the runtime like the
// tensor-map encoder (no link against libcuda).
using PfnCtxGetCurrent = CUresult (*)(CUcontext*);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long*);

struct CtxApi {
    PfnCtxGetCurrent get_current = nullptr;
    PfnCtxGetId get_id = nullptr;
};
const CtxApi& ctx_api() {
    static std::once_flag once;
    static CtxApi api;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            api.get_current = reinterpret_cast<PfnCtxGetCurrent>(f);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            api.get_id = reinterpret_cast<PfnCtxGetId>(f);
        cudaGetLastError();
    });
    return api;
}

// Device address of g_noalloc_scratch in the current CUDA context.  The
// address belongs to the module image loaded in one context: a context the
// caller made current, or the primary context created again after
// cudaDeviceReset, has its own.  So it is looked up once per context, keyed
// by the context's process-unique id, and kept; without the id query it is
// looked up on every call.
mm_status noalloc_scratch(void** out) {
    // the lookup itself makes the runtime's context current if none is yet
    void* p = nullptr;
    const CtxApi& api = ctx_api();
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    const bool keyed = api.get_current && api.get_id && api.get_current(&ctx) == CUDA_SUCCESS && ctx &&
                       api.get_id(ctx, &id) == CUDA_SUCCESS;
    static std::mutex mu;
    constexpr int kSlots = 64;
    static unsigned long long ids[kSlots] = {};
    static void* addrs[kSlots] = {};
    static int next = 0;
    if (keyed) {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < kSlots; ++i)
            if (ids[i] == id && addrs[i]) { *out = addrs[i]; return MM_OK; }
    }
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return MM_ERR_CUDA;
    }
    if (keyed) {
        std::lock_guard<std::mutex> lock(mu);
        ids[next] = id;
        addrs[next] = p;
        next = (next + 1) % kSlots;
    }
    *out = p;
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
        case MM_ERR_TIMEOUT:
            return "a kernel of the call gave up waiting (for its bulk copies, or for a chunk summary that was "
                   "never written); its outputs are not valid";
        case MM_ERR_ARG: return "an argument value is out of range (norm_eps must be positive and finite)";
        case MM_ERR_BOUNDS: return "a kernel of the checked build skipped an access outside its buffer";
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
    if (v & mm::kFaultBounds) return MM_ERR_BOUNDS;
    return v ? MM_ERR_TIMEOUT : MM_OK;
}

mm_status mamba_check_status(const void* workspace, void* stream) {
    const void* ws = workspace;
    if (!ws) {
        void* p = nullptr;
        if (mm_status st = noalloc_scratch(&p); st != MM_OK) return st;
        ws = p;
    }
    if (!aligned16(ws)) return MM_ERR_ALIGN;
    unsigned long long hdr[2] = {0, 0};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(hdr, ws, sizeof(hdr), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return MM_ERR_CUDA;
    }
    if ((hdr[0] & 0xff) == 0 || (hdr[0] >> 8) != hdr[1]) return MM_OK;
    return (hdr[0] & 0xff) == mm::kStatusBounds ? MM_ERR_BOUNDS : MM_ERR_TIMEOUT;
}

size_t mamba_mixer_workspace_size(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state,
                                  int64_t d_conv, mm_dtype act) {
    if ((act != MM_F32 && act != MM_BF16) || batch <= 0 || seqlen < 0 || d_inner <= 0 || d_state != 16 ||
        d_conv != 4 || d_inner % 8 != 0 || d_inner > (1 << 24) || batch > (1 << 24) ||
        !seqlen_ok(seqlen, d_inner, act == MM_F32 ? 4 : 2))
        return 0;
    return plan_fwd(batch, seqlen, d_inner, plan_sms()).ws_bytes;
}

}  // extern "C"

namespace {

// mamba_mixer_fwd and mamba_mixer_fwd_normed: validate, check the workspace, launch.
mm_status fwd_with_workspace(const FwdArgs& a, void* workspace, size_t workspace_bytes, void* stream) {
    const int64_t batch = a.batch, seqlen = a.seqlen, d_inner = a.d_inner;
    FwdBytes nb;
    if (mm_status st = validate_fwd(a, &nb); st != MM_OK) return st;
    if (batch == 0) return MM_OK;
    const int sms = plan_sms();
    const FwdPlan pl = plan_fwd(batch, seqlen, d_inner, sms);
    if (!workspace || workspace_bytes < pl.ws_bytes) return MM_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MM_ERR_ALIGN;
    if (workspace_overlaps(a, nb, workspace, pl.ws_bytes)) return MM_ERR_ALIAS;
    if (mm_status st = check_device(); st != MM_OK) return st;
    return run_fwd(a, pl, sms, workspace, next_call_id(), static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

mm_status mamba_mixer_fwd(const void* xz, const float* conv_w, const float* conv_b,
                          const void* dt, const float* dt_bias, const float* A,
                          const void* Bm, const void* Cm, const float* Dskip,
                          const float* h0, const void* conv_state_in,
                          void* y, float* h_last, void* conv_state_out,
                          int64_t batch, int64_t seqlen, int64_t d_inner,
                          int64_t d_state, int64_t d_conv, mm_dtype act,
                          void* workspace, size_t workspace_bytes, void* stream)
{
    const FwdArgs a{xz, conv_w, conv_b, dt, dt_bias, A, Bm, Cm, Dskip, h0, conv_state_in, y, h_last,
                    conv_state_out, batch, seqlen, d_inner, d_state, d_conv, act};
    return fwd_with_workspace(a, workspace, workspace_bytes, stream);
}

mm_status mamba_mixer_fwd_normed(const void* xz, const float* conv_w, const float* conv_b,
                                 const void* dt, const float* dt_bias, const float* A,
                                 const void* Bm, const void* Cm, const float* Dskip,
                                 const float* h0, const void* conv_state_in,
                                 void* y, float* h_last, void* conv_state_out,
                                 int64_t batch, int64_t seqlen, int64_t d_inner,
                                 int64_t d_state, int64_t d_conv, mm_dtype act,
                                 const float* b_norm_w, const float* c_norm_w, float norm_eps,
                                 void* workspace, size_t workspace_bytes, void* stream)
{
    FwdArgs a{xz, conv_w, conv_b, dt, dt_bias, A, Bm, Cm, Dskip, h0, conv_state_in, y, h_last,
              conv_state_out, batch, seqlen, d_inner, d_state, d_conv, act};
    a.b_norm_w = b_norm_w;
    a.c_norm_w = c_norm_w;
    a.norm_eps = norm_eps;
    return fwd_with_workspace(a, workspace, workspace_bytes, stream);
}

}  // extern "C"

namespace {

mm_status state_update_impl(const void* x, const void* z, const void* dt,
                            const float* conv_w, const float* conv_b,
                            const float* dt_bias, const float* Dskip, const float* A,
                            const void* Bm, const void* Cm,
                            float* ssm_state, void* conv_state, void* y,
                            int64_t n_layers, int64_t batch, int64_t d_inner,
                            int64_t d_state, int64_t d_conv, mm_dtype act,
                            const float* b_norm_w, const float* c_norm_w, float norm_eps, void* stream)
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
    if ((b_norm_w || c_norm_w) && !(norm_eps > 0.0f && norm_eps < 1e30f)) return MM_ERR_ARG;
    const void* all[] = {x, z, dt, conv_w, conv_b, dt_bias, Dskip, A, Bm, Cm, ssm_state, conv_state, y,
                         b_norm_w, c_norm_w};
    for (const void* q : all)
        if (q && !aligned16(q)) return MM_ERR_ALIGN;

    const int64_t tok_bytes = rows * es;
    const int64_t par = n_layers * d_inner * 4;
    const Span in[] = {span(x, tok_bytes), span(z, tok_bytes), span(dt, tok_bytes),
                       span(conv_w, par * d_conv), span(conv_b, par), span(dt_bias, par), span(Dskip, par),
                       span(A, par * d_state), span(Bm, lb * d_state * es), span(Cm, lb * d_state * es),
                       span(b_norm_w, n_layers * d_state * 4), span(c_norm_w, n_layers * d_state * 4)};
    const Span io[] = {span(ssm_state, st_bytes), span(conv_state, rows * (d_conv - 1) * es), span(y, tok_bytes)};
    for (const Span& o : io)
        for (const Span& i : in)
            if (overlaps(o, i)) return MM_ERR_ALIAS;
    if (overlaps(io[0], io[1]) || overlaps(io[0], io[2]) || overlaps(io[1], io[2])) return MM_ERR_ALIAS;

    if (mm_status st = check_device(); st != MM_OK) return st;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const unsigned grid = static_cast<unsigned>((warps + 7) / 8);
    auto launch = [&](auto tag_t, auto math, auto norm) {
        using T = decltype(tag_t);
        constexpr bool NORM = decltype(norm)::value;
        mm::state_update_kernel<T, decltype(math), NORM><<<grid, 256, 0, s>>>(
            static_cast<const T*>(x), static_cast<const T*>(z), static_cast<const T*>(dt), conv_w, conv_b,
            dt_bias, Dskip, A, static_cast<const T*>(Bm), static_cast<const T*>(Cm), ssm_state,
            static_cast<T*>(conv_state), static_cast<T*>(y), static_cast<int>(n_layers), static_cast<int>(batch),
            static_cast<int>(d_inner), b_norm_w, c_norm_w, norm_eps);
    };
    const bool norm = b_norm_w || c_norm_w;
    if (act == MM_BF16) {
        if (norm) launch(__nv_bfloat16{}, mm::MathFast{}, std::true_type{});
        else launch(__nv_bfloat16{}, mm::MathFast{}, std::false_type{});
    } else {
        if (norm) launch(float{}, mm::MathExact{}, std::true_type{});
        else launch(float{}, mm::MathExact{}, std::false_type{});
    }
    if (cudaGetLastError() != cudaSuccess) return MM_ERR_CUDA;
    return MM_OK;
}

}  // namespace

extern "C" {

mm_status mamba_state_update(const void* x, const void* z, const void* dt,
                             const float* conv_w, const float* conv_b,
                             const float* dt_bias, const float* Dskip, const float* A,
                             const void* Bm, const void* Cm,
                             float* ssm_state, void* conv_state, void* y,
                             int64_t n_layers, int64_t batch, int64_t d_inner,
                             int64_t d_state, int64_t d_conv, mm_dtype act, void* stream)
{
    return state_update_impl(x, z, dt, conv_w, conv_b, dt_bias, Dskip, A, Bm, Cm, ssm_state, conv_state, y,
                             n_layers, batch, d_inner, d_state, d_conv, act, nullptr, nullptr, 0.0f, stream);
}

mm_status mamba_state_update_normed(const void* x, const void* z, const void* dt,
                                    const float* conv_w, const float* conv_b,
                                    const float* dt_bias, const float* Dskip, const float* A,
                                    const void* Bm, const void* Cm,
                                    float* ssm_state, void* conv_state, void* y,
                                    int64_t n_layers, int64_t batch, int64_t d_inner,
                                    int64_t d_state, int64_t d_conv, mm_dtype act,
                                    const float* b_norm_w, const float* c_norm_w, float norm_eps, void* stream)
{
    return state_update_impl(x, z, dt, conv_w, conv_b, dt_bias, Dskip, A, Bm, Cm, ssm_state, conv_state, y,
                             n_layers, batch, d_inner, d_state, d_conv, act, b_norm_w, c_norm_w, norm_eps, stream);
}

mm_status mamba_mixer_fwd_noalloc(const void* xz, const float* conv_w, const float* conv_b,
                                  const void* dt, const float* dt_bias, const float* A,
                                  const void* Bm, const void* Cm, const float* Dskip,
                                  const float* h0, const void* conv_state_in,
                                  void* y, float* h_last, void* conv_state_out,
                                  int64_t batch, int64_t seqlen, int64_t d_inner,
                                  int64_t d_state, int64_t d_conv, mm_dtype act, void* stream)
{
    const FwdArgs a{xz, conv_w, conv_b, dt, dt_bias, A, Bm, Cm, Dskip, h0, conv_state_in, y, h_last,
                    conv_state_out, batch, seqlen, d_inner, d_state, d_conv, act};
    FwdBytes nb;
    if (mm_status st = validate_fwd(a, &nb); st != MM_OK) return st;
    if (batch == 0) return MM_OK;
    const int sms = plan_sms();
    const FwdPlan pl = plan_fwd(batch, seqlen, d_inner, sms);
    if (pl.ws_bytes > MAMBA_MIXER_NOALLOC_SCRATCH_BYTES) return MM_ERR_SCRATCH_LIMIT;
    if (mm_status st = check_device(); st != MM_OK) return st;
    void* scratch = nullptr;
    if (mm_status st = noalloc_scratch(&scratch); st != MM_OK) return st;
    return run_fwd(a, pl, sms, scratch, next_call_id(), static_cast<cudaStream_t>(stream));
}

size_t mamba_mixer_host_workspace_size(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state,
                                       int64_t d_conv, mm_dtype act) {
    if ((act != MM_F32 && act != MM_BF16) || batch <= 0 || seqlen < 0 || d_inner <= 0 || d_state != 16 ||
        d_conv != 4 || d_inner % 8 != 0 || d_inner > (1 << 24) || batch > (1 << 24))
        return 0;
    int64_t tokens, bytes;
    if (!mul_ok(batch, seqlen, &tokens) || !mul_ok(tokens, 2 * d_inner * 4, &bytes)) return 0;
    const int64_t es = act == MM_F32 ? 4 : 2;
    const HostPlan hp = plan_host(batch, seqlen, d_inner, es, plan_sms());
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
    const FwdArgs a{xz, conv_w, conv_b, dt, dt_bias, A, Bm, Cm, Dskip, h0, conv_state_in, y, h_last,
                    conv_state_out, batch, seqlen, d_inner, d_state, d_conv, act};
    FwdBytes nb;
    if (mm_status st = check_sizes(a, &nb); st != MM_OK) return st;
    if (batch == 0) return MM_OK;

    if (!conv_w || !dt_bias || !A || !h_last || !conv_state_out) return MM_ERR_NULL;
    if (seqlen > 0 && (!xz || !dt || !Bm || !Cm || !y)) return MM_ERR_NULL;
    // device pointers and the workspace: 16-byte aligned (host buffers need not be)
    const void* dev_ptrs[] = {conv_w, conv_b, dt_bias, A, Dskip};
    for (const void* q : dev_ptrs)
        if (q && !aligned16(q)) return MM_ERR_ALIGN;
    // host outputs may not overlap host inputs
    const Span in[] = {span(xz, nb.xz), span(dt, nb.dt), span(Bm, nb.bc), span(Cm, nb.bc),
                       span(h0, nb.st), span(conv_state_in, nb.cs)};
    const Span out[] = {span(y, nb.dt), span(h_last, nb.st), span(conv_state_out, nb.cs)};
    for (const Span& o : out)
        for (const Span& i : in)
            if (overlaps(o, i)) return MM_ERR_ALIAS;
    if (overlaps(out[0], out[1]) || overlaps(out[0], out[2]) || overlaps(out[1], out[2])) return MM_ERR_ALIAS;

    const int64_t es = nb.es;
    const int sms = plan_sms();
    const HostPlan hp = plan_host(batch, seqlen, d_inner, es, sms);
    if (!seqlen_ok(hp.piece, d_inner, es)) return MM_ERR_SHAPE;   // each piece is one device call
    if (!workspace || workspace_bytes < hp.total) return MM_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MM_ERR_ALIGN;
    // the device parameters may not overlap the workspace the pieces are staged in
    {
        const Span w = span(workspace, static_cast<int64_t>(hp.total));
        const Span par[] = {span(conv_w, d_inner * d_conv * 4), span(conv_b, d_inner * 4),
                            span(dt_bias, d_inner * 4), span(A, d_inner * d_state * 4), span(Dskip, d_inner * 4)};
        for (const Span& q : par)
            if (overlaps(w, q)) return MM_ERR_ALIAS;
    }
    if (mm_status st = check_device(); st != MM_OK) return st;

    cudaStream_t sc = static_cast<cudaStream_t>(stream);
    cudaStream_t s_in = static_cast<cudaStream_t>(h2d_stream);
    cudaStream_t s_out = static_cast<cudaStream_t>(d2h_stream);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    void* fwd_ws = ws;
    unsigned char* slot[2] = {ws + hp.fwd_ws, ws + hp.fwd_ws + hp.slot};
    unsigned char* carry[2] = {ws + hp.fwd_ws + 2 * hp.slot, ws + hp.fwd_ws + 2 * hp.slot + hp.carry};
    // every piece records its failures under the call's one epoch, so the
    // workspace's status reports a failure of any piece
    const unsigned long long epoch = next_call_id();

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
    if (h0) chk(cudaMemcpyAsync(carry[0], h0, static_cast<size_t>(nb.st), cudaMemcpyHostToDevice, s_in));
    if (conv_state_in)
        chk(cudaMemcpyAsync(carry[0] + hp.carry_h, conv_state_in, static_cast<size_t>(nb.cs),
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
        if (!ok) break;
        const FwdArgs pa{sl, conv_w, conv_b, sl + hp.off_dt, dt_bias, A, sl + hp.off_b, sl + hp.off_c, Dskip,
                         (first && !h0) ? nullptr : reinterpret_cast<const float*>(cin),
                         (first && !conv_state_in) ? nullptr : cin + hp.carry_h, sl + hp.off_y,
                         reinterpret_cast<float*>(cout), cout + hp.carry_h, batch, static_cast<int64_t>(n),
                         d_inner, d_state, d_conv, act};
        fwd_status = run_fwd(pa, plan_fwd(batch, static_cast<int64_t>(n), d_inner, sms), sms, fwd_ws, epoch, sc);
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
        chk(cudaMemcpyAsync(h_last, cl, static_cast<size_t>(nb.st), cudaMemcpyDeviceToHost, s_out));
        chk(cudaMemcpyAsync(conv_state_out, cl + hp.carry_h, static_cast<size_t>(nb.cs),
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

// ---------------------------------------------------------------- projections (tcgen05 GEMM)
namespace {

// 2-D map over a row-major [rows][cols] bf16 matrix, [box_rows][64] boxes,
// 128-byte swizzle (the layout the MMA's shared-memory descriptor reads).
bool encode_gemm_2d(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * 2)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(mm::kGemmBK), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tile width of the GEMM for N output columns: one tile up to 144 columns
// (x_proj's 288 = 2 x 144), else 256-column tiles.
int gemm_bn(int64_t N) { return N <= 64 ? 64 : N <= 128 ? 128 : (N <= 144 || N == 288) ? 144 : 256; }

// Map of a bf16 output [M][N] (rows ldo elements apart) in 64-column x
// 32-row boxes with the 128-byte swizzle: the GEMM's staged epilogue.
bool encode_gemm_out(CUtensorMap* m, void* base, int64_t cols, int64_t rows, int64_t ldo) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldo * 2)};
    const cuuint32_t box[2] = {64, 32};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int NSUB, int STAGES, bool OUT_BF16>
cudaError_t launch_gemm_t(mm::GemmParams gp, const void* A, const void* W, int ksplit, cudaStream_t s) {
    CUtensorMap ta, tw, to;
    if (!encode_gemm_2d(&ta, A, gp.K, gp.M, mm::kGemmBM) || !encode_gemm_2d(&tw, W, gp.K, gp.N, BN))
        return cudaErrorInvalidValue;
    // bf16 tiles of whole 64-column boxes go out by bulk tensor stores when the
    // rows are 16-byte multiples (MAMBA_MIXER_GEMM_ROW_STORES=1 keeps the
    // per-thread row stores, for comparison)
    std::memset(&to, 0, sizeof(to));
    gp.tma_out = 0;
    if (OUT_BF16 && NSUB == 1 && BN % 64 == 0 && gp.ldo % 8 == 0 && gp.M > 0 &&
        env_int("MAMBA_MIXER_GEMM_ROW_STORES", 1, 1) == 0) {
        gp.tma_out = encode_gemm_out(&to, gp.out, gp.N, gp.M, gp.ldo) ? 1 : 0;   // else the row stores
    }
    auto kern = mm::proj_gemm_kernel<BN, NSUB, STAGES, OUT_BF16>;
    const int smem = mm::GemmLayout<BN, NSUB>::smem_bytes(STAGES);
    static std::atomic<unsigned long long> smem_allowed{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaGetLastError();
    const unsigned long long bit = dev < 64 ? 1ull << dev : 0;
    if (!(bit && (smem_allowed.load() & bit))) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        if (bit) smem_allowed.fetch_or(bit);
    }
    const dim3 grid(static_cast<unsigned>((gp.M + mm::kGemmBM - 1) / mm::kGemmBM),
                    static_cast<unsigned>((gp.N + BN * NSUB - 1) / (BN * NSUB)), static_cast<unsigned>(ksplit));
    kern<<<grid, mm::kGemmThreads, forced_launch_failure() ? (1 << 20) : smem, s>>>(gp, ta, tw, to);
    return cudaGetLastError();
}

// Shapes: up to 128 outputs, one sub-tile; 288 (x_proj), two 144-wide
// sub-tiles sharing each A tile; otherwise 256-wide tiles.  A product with
// few K tiles per CTA (dt_proj: 4) takes a 2-deep ring, so two CTAs share an
// SM and one's epilogue overlaps the other's copies and MMAs.
template <bool OUT_BF16>
cudaError_t launch_gemm(mm::GemmParams gp, const void* A, const void* W, int ksplit, cudaStream_t s) {
    const bool short_k = gp.k_tiles_per_split <= 4;
    switch (gemm_bn(gp.N)) {
        case 64: return launch_gemm_t<64, 1, 8, OUT_BF16>(gp, A, W, ksplit, s);
        case 128: return launch_gemm_t<128, 1, 6, OUT_BF16>(gp, A, W, ksplit, s);
        case 144: return gp.N > 144 ? launch_gemm_t<144, 2, 4, OUT_BF16>(gp, A, W, ksplit, s)
                                    : launch_gemm_t<144, 1, 6, OUT_BF16>(gp, A, W, ksplit, s);
        default: return short_k ? launch_gemm_t<256, 1, 2, OUT_BF16>(gp, A, W, ksplit, s)
                                : launch_gemm_t<256, 1, 4, OUT_BF16>(gp, A, W, ksplit, s);
    }
}

// Split of K for a product: until the grid covers the SMs once (its CTAs each
// fill an SM's shared memory with their ring), at most 16 ways and at least
// 8 K tiles per CTA.
int gemm_ksplit(int64_t M, int64_t N, int64_t K, int sms) {
    const int64_t m_tiles = (M + mm::kGemmBM - 1) / mm::kGemmBM;
    const int bn = gemm_bn(N);
    const int64_t n_groups = N == 288 ? 1 : (N + bn - 1) / bn;
    const int64_t k_tiles = (K + mm::kGemmBK - 1) / mm::kGemmBK;
    const int64_t split = std::max<int64_t>(1, sms / std::max<int64_t>(1, m_tiles * n_groups));
    return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>({split, k_tiles / 8, 16})));
}

size_t matmul_ws_bytes(int64_t M, int64_t N, int64_t K, int sms) {
    const int ks = gemm_ksplit(M, N, K, sms);
    return kWsHeader + (ks > 1 ? align256(static_cast<size_t>(ks) * M * N * 4) : 0);
}


// Plan of the mixer with its projections: regions of its workspace (each
// 256-byte aligned; the scan's own workspace first, so mamba_check_status
// reads the call's status at the workspace's start) and x_proj's split.
struct ProjPlan {
    FwdPlan scan;
    int64_t M = 0;          // tokens (batch x seqlen)
    int R = 0, NC = 0;      // dt_rank, x_proj's output width R + 2 d_state
    int ksplit = 1;
    size_t off_u = 0, off_part = 0, off_dtlow = 0, off_b = 0, off_c = 0, off_dt = 0, total = 0;
};

ProjPlan plan_projected(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t dt_rank, int sms) {
    ProjPlan pp;
    pp.scan = plan_fwd(batch, seqlen, d_inner, sms);
    pp.M = batch * seqlen;
    pp.R = static_cast<int>(dt_rank);
    pp.NC = pp.R + 32;
    pp.ksplit = gemm_ksplit(pp.M, pp.NC, d_inner, sms);
    const size_t M = static_cast<size_t>(pp.M), D = static_cast<size_t>(d_inner);
    pp.off_u = align256(pp.scan.ws_bytes);
    pp.off_part = pp.off_u + align256(M * D * 2);
    pp.off_dtlow = pp.off_part + align256(static_cast<size_t>(pp.ksplit) * M * pp.NC * 4);
    pp.off_b = pp.off_dtlow + align256(M * pp.R * 2);
    pp.off_c = pp.off_b + align256(M * 16 * 2);
    pp.off_dt = pp.off_c + align256(M * 16 * 2);
    pp.total = pp.off_dt + align256(M * D * 2);
    return pp;
}

bool proj_sizes_ok(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state, int64_t dt_rank,
                   int64_t d_conv) {
    int64_t tokens;
    return batch >= 0 && seqlen >= 0 && d_inner > 0 && d_state == 16 && d_conv == 4 && d_inner % 64 == 0 &&
           d_inner <= (1 << 20) && dt_rank > 0 && dt_rank % 32 == 0 && dt_rank <= 1024 &&
           mul_ok(batch, seqlen, &tokens) && tokens < (int64_t(1) << 31) && seqlen_ok(seqlen, d_inner, 2);
}

}  // namespace

extern "C" {

size_t mamba_proj_matmul_workspace_size(int64_t M, int64_t N, int64_t K) {
    if (M <= 0 || N <= 0 || K <= 0 || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
        return 0;
    return matmul_ws_bytes(M, N, K, plan_sms());
}

mm_status mamba_proj_matmul(const void* A, const void* W, void* out, int64_t M, int64_t N, int64_t K,
                            mm_dtype out_dtype, void* workspace, size_t workspace_bytes, void* stream)
{
    if (out_dtype != MM_F32 && out_dtype != MM_BF16) return MM_ERR_DTYPE;
    if (M < 0 || N <= 0 || K <= 0 || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
        return MM_ERR_SHAPE;
    if (K % 8 != 0 || N % 8 != 0) return MM_ERR_UNSUPPORTED;
    if (M == 0) return MM_OK;
    if (!A || !W || !out) return MM_ERR_NULL;
    if (!aligned16(A) || !aligned16(W) || !aligned16(out)) return MM_ERR_ALIGN;
    const int64_t es = out_dtype == MM_F32 ? 4 : 2;
    const Span a = span(A, M * K * 2), w = span(W, N * K * 2), o = span(out, M * N * es);
    if (overlaps(o, a) || overlaps(o, w)) return MM_ERR_ALIAS;
    const int sms = plan_sms();
    const size_t need = matmul_ws_bytes(M, N, K, sms);
    if (!workspace || workspace_bytes < need) return MM_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MM_ERR_ALIGN;
    const Span ws = span(workspace, static_cast<int64_t>(need));
    if (overlaps(ws, a) || overlaps(ws, w) || overlaps(ws, o)) return MM_ERR_ALIAS;
    if (mm_status st = check_device(); st != MM_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the call's status: the GEMM writes the epoch into hdr[1]
    const unsigned long long epoch = next_call_id();
    unsigned long long* hdr = static_cast<unsigned long long*>(workspace);
    // a tall, narrow product is split in K: fp32 partials in the workspace,
    // then summed into `out`
    const int ks = gemm_ksplit(M, N, K, sms);
    float* part = ks > 1 ? reinterpret_cast<float*>(static_cast<unsigned char*>(workspace) + kWsHeader) : nullptr;
    const int k_tiles = static_cast<int>((K + mm::kGemmBK - 1) / mm::kGemmBK);
    mm::GemmParams gp{};
    gp.out = ks > 1 ? static_cast<void*>(part) : out;
    gp.ldo = N;
    gp.split_stride = M * N;
    gp.M = static_cast<int>(M);
    gp.N = static_cast<int>(N);
    gp.K = static_cast<int>(K);
    gp.k_tiles_per_split = (k_tiles + ks - 1) / ks;
    gp.wait_limit = copy_wait_limit();
    gp.status = hdr;
    gp.status_epoch = epoch;
    cudaError_t e = (out_dtype == MM_BF16 && ks == 1) ? launch_gemm<true>(gp, A, W, 1, s)
                                                       : launch_gemm<false>(gp, A, W, ks, s);
    if (e == cudaSuccess && ks > 1) {
        const int64_t n = M * N;
        const unsigned blocks = static_cast<unsigned>((n / 4 + 255) / 256);
        if (out_dtype == MM_BF16) mm::splitk_reduce_kernel<true><<<blocks, 256, 0, s>>>(part, ks, n, out);
        else mm::splitk_reduce_kernel<false><<<blocks, 256, 0, s>>>(part, ks, n, out);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) { cudaGetLastError(); return MM_ERR_CUDA; }
    return MM_OK;
}

mm_status mamba_mixer_projected_layout(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state,
                                       int64_t dt_rank, int64_t d_conv, size_t offsets[5]) {
    if (!offsets) return MM_ERR_NULL;
    if (batch <= 0 || !proj_sizes_ok(batch, seqlen, d_inner, d_state, dt_rank, d_conv)) return MM_ERR_SHAPE;
    const ProjPlan pp = plan_projected(batch, seqlen, d_inner, dt_rank, plan_sms());
    offsets[0] = pp.off_u;
    offsets[1] = pp.off_dtlow;
    offsets[2] = pp.off_b;
    offsets[3] = pp.off_c;
    offsets[4] = pp.off_dt;
    return MM_OK;
}

size_t mamba_mixer_projected_workspace_size(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state,
                                            int64_t dt_rank, int64_t d_conv, mm_dtype act) {
    if (act != MM_BF16 || batch <= 0 || !proj_sizes_ok(batch, seqlen, d_inner, d_state, dt_rank, d_conv)) return 0;
    return plan_projected(batch, seqlen, d_inner, dt_rank, plan_sms()).total;
}

mm_status mamba_mixer_fwd_projected(const void* xz, const float* conv_w, const float* conv_b,
                                    const void* W_x, const void* W_dt, const float* dt_bias, const float* A,
                                    const float* Dskip, const float* h0, const void* conv_state_in,
                                    const float* dt_norm_w, const float* b_norm_w, const float* c_norm_w,
                                    float norm_eps, void* y, float* h_last, void* conv_state_out,
                                    int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state,
                                    int64_t dt_rank, int64_t d_conv, mm_dtype act,
                                    void* workspace, size_t workspace_bytes, void* stream)
{
    if (act != MM_F32 && act != MM_BF16) return MM_ERR_DTYPE;
    if (act != MM_BF16) return MM_ERR_UNSUPPORTED;        // the tensor-core products take bf16 operands
    if (batch < 0 || seqlen < 0 || d_inner <= 0 || d_state <= 0 || dt_rank <= 0 || d_conv <= 0) return MM_ERR_SHAPE;
    if (!proj_sizes_ok(batch, seqlen, d_inner, d_state, dt_rank, d_conv)) {
        if (d_state != 16 || d_conv != 4 || d_inner % 64 != 0 || dt_rank % 32 != 0) return MM_ERR_UNSUPPORTED;
        return MM_ERR_SHAPE;
    }
    if (batch == 0) return MM_OK;
    if (!W_x || !W_dt) return MM_ERR_NULL;
    if (!aligned16(W_x) || !aligned16(W_dt)) return MM_ERR_ALIGN;
    if ((dt_norm_w || b_norm_w || c_norm_w) && !(norm_eps > 0.0f && norm_eps < 1e30f)) return MM_ERR_ARG;
    for (const void* q : {static_cast<const void*>(dt_norm_w), static_cast<const void*>(b_norm_w),
                          static_cast<const void*>(c_norm_w)})
        if (q && !aligned16(q)) return MM_ERR_ALIGN;
    const int sms = plan_sms();
    const ProjPlan pp = plan_projected(batch, seqlen, d_inner, dt_rank, sms);
    if (!workspace || workspace_bytes < pp.total) return MM_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MM_ERR_ALIGN;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    __nv_bfloat16* u = reinterpret_cast<__nv_bfloat16*>(ws + pp.off_u);
    float* part = reinterpret_cast<float*>(ws + pp.off_part);
    __nv_bfloat16* dtlow = reinterpret_cast<__nv_bfloat16*>(ws + pp.off_dtlow);
    __nv_bfloat16* Bm = reinterpret_cast<__nv_bfloat16*>(ws + pp.off_b);
    __nv_bfloat16* Cm = reinterpret_cast<__nv_bfloat16*>(ws + pp.off_c);
    __nv_bfloat16* dt = reinterpret_cast<__nv_bfloat16*>(ws + pp.off_dt);
    // the scan's arguments, validated as one mamba_mixer_fwd_normed call on the
    // workspace's intermediates (B and C are already normalised by x_proj's epilogue)
    const FwdArgs a{xz, conv_w, conv_b, dt, dt_bias, A, Bm, Cm, Dskip, h0, conv_state_in, y, h_last,
                    conv_state_out, batch, seqlen, d_inner, d_state, d_conv, act};
    FwdBytes nb;
    if (mm_status st = validate_fwd(a, &nb); st != MM_OK) return st;
    // the weights and the caller's buffers may not overlap the workspace
    {
        const Span w = span(workspace, static_cast<int64_t>(pp.total));
        const int64_t NC = pp.NC;
        const Span ins[] = {span(xz, nb.xz), span(conv_w, d_inner * d_conv * 4), span(conv_b, d_inner * 4),
                            span(W_x, NC * d_inner * 2), span(W_dt, d_inner * dt_rank * 2), span(dt_bias, d_inner * 4),
                            span(A, d_inner * d_state * 4), span(Dskip, d_inner * 4), span(h0, nb.st),
                            span(conv_state_in, nb.cs), span(dt_norm_w, dt_rank * 4), span(b_norm_w, 64),
                            span(c_norm_w, 64), span(y, nb.dt), span(h_last, nb.st), span(conv_state_out, nb.cs)};
        for (const Span& q : ins)
            if (overlaps(w, q)) return MM_ERR_ALIAS;
        const Span outs[] = {span(y, nb.dt), span(h_last, nb.st), span(conv_state_out, nb.cs)};
        for (const Span& o : outs)
            if (overlaps(o, span(W_x, NC * d_inner * 2)) || overlaps(o, span(W_dt, d_inner * dt_rank * 2)) ||
                overlaps(o, span(dt_norm_w, dt_rank * 4)))
                return MM_ERR_ALIAS;
    }
    if (mm_status st = check_device(); st != MM_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const unsigned long long epoch = next_call_id();
    unsigned long long* hdr = reinterpret_cast<unsigned long long*>(ws);
    if (seqlen > 0) {
        const int64_t M = pp.M;
        // u = SiLU(conv(x))
        {
            const dim3 grid(static_cast<unsigned>((d_inner / 8 + 127) / 128),
                            static_cast<unsigned>((seqlen + mm::kConvTokens - 1) / mm::kConvTokens),
                            static_cast<unsigned>(batch));
            mm::conv_silu_kernel<<<grid, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(xz), conv_w, conv_b,
                                                      static_cast<const __nv_bfloat16*>(conv_state_in), u, seqlen,
                                                      static_cast<int>(d_inner));
            if (cudaGetLastError() != cudaSuccess) return MM_ERR_CUDA;
        }
        // x_proj partials: [ksplit][M][R + 32] fp32
        mm::GemmParams gp{};
        gp.out = part;
        gp.ldo = pp.NC;
        gp.split_stride = M * pp.NC;
        gp.M = static_cast<int>(M);
        gp.N = pp.NC;
        gp.K = static_cast<int>(d_inner);
        const int k_tiles = static_cast<int>((d_inner + mm::kGemmBK - 1) / mm::kGemmBK);
        gp.k_tiles_per_split = (k_tiles + pp.ksplit - 1) / pp.ksplit;
        gp.wait_limit = copy_wait_limit();
        gp.status = hdr;
        gp.status_epoch = epoch;
        if (launch_gemm<false>(gp, u, W_x, pp.ksplit, s) != cudaSuccess) { cudaGetLastError(); return MM_ERR_CUDA; }
        // sum the partials; split into dt_low | B | C, normalised, bf16
        mm::xproj_epilogue_kernel<<<static_cast<unsigned>((M + 7) / 8), 256, 0, s>>>(
            part, pp.ksplit, gp.split_stride, M, pp.R, dt_norm_w, b_norm_w, c_norm_w, norm_eps, dtlow, Bm, Cm);
        if (cudaGetLastError() != cudaSuccess) return MM_ERR_CUDA;
        // dt = dt_low W_dt^T: [M][d_inner] bf16
        mm::GemmParams gd{};
        gd.out = dt;
        gd.ldo = d_inner;
        gd.M = static_cast<int>(M);
        gd.N = static_cast<int>(d_inner);
        gd.K = pp.R;
        gd.k_tiles_per_split = (pp.R + mm::kGemmBK - 1) / mm::kGemmBK;
        gd.wait_limit = gp.wait_limit;
        gd.status = hdr;
        gd.status_epoch = epoch;
        if (launch_gemm<true>(gd, dtlow, W_dt, 1, s) != cudaSuccess) { cudaGetLastError(); return MM_ERR_CUDA; }
    }
    // the selective scan on (x, z, dt, B, C)
    return run_fwd(a, pp.scan, sms, workspace, epoch, s);
}

}  // extern "C"


// ---------------------------------------------------------------- Mamba-2 form (tcgen05 chunked scan)
namespace {

// Workspace of mamba_ssd_fwd (every region 256-byte aligned):
//   header [256 B]                        the call status
//   S      [B][chunks][H][P][N] f32       chunk states from zero
//   Hin    [2][B][chunks][H][P][N] bf16   state entering each chunk: hi parts, then lo parts
//   dec    [B][H][chunks] f32             each chunk's total decay
struct SsdPlan {
    int64_t chunks = 0;
    size_t off_s = 0, off_hin = 0, off_dec = 0, total = 0;
};

SsdPlan plan_ssd(int64_t batch, int64_t seqlen, int64_t heads) {
    SsdPlan pl;
    pl.chunks = (seqlen + mm::kSsdQ - 1) / mm::kSsdQ;
    const size_t states = static_cast<size_t>(batch) * pl.chunks * heads * mm::kSsdP * mm::kSsdN;
    pl.off_s = kWsHeader;
    pl.off_hin = pl.off_s + align256(states * 4);
    pl.off_dec = pl.off_hin + align256(states * 2 * 2);
    pl.total = pl.off_dec + align256(static_cast<size_t>(batch) * heads * pl.chunks * 4);
    return pl;
}

// Sizes the kernels address: grid y/z limits, 32-bit tensor-copy coordinates
// (tokens, and rows of the [2 * B * chunks * H * P][N] state copies).
bool ssd_sizes_ok(int64_t batch, int64_t seqlen, int64_t heads, int64_t groups) {
    if (batch < 0 || seqlen < 0 || heads <= 0 || groups <= 0 || heads % groups != 0) return false;
    if (batch > 65535 || heads > 65535 || seqlen >= (int64_t(1) << 31) - mm::kSsdQ) return false;
    const int64_t chunks = (seqlen + mm::kSsdQ - 1) / mm::kSsdQ;
    int64_t rows;
    return mul_ok(batch * chunks, heads * mm::kSsdP, &rows) && 2 * rows < (int64_t(1) << 31) &&
           seqlen * heads * mm::kSsdP * 2 < (int64_t(1) << 40);
}

// 3-D map over a bf16 [batch][rows][cols] tensor, [box_rows][64] boxes with
// the 128-byte swizzle of the products' operand tiles.
bool encode_sw128_3d(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int64_t batch, int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                                static_cast<cuuint64_t>(batch)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols * 2), static_cast<cuuint64_t>(rows * cols * 2)};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" {

size_t mamba_ssd_workspace_size(int64_t batch, int64_t seqlen, int64_t heads, int64_t headdim, int64_t d_state,
                                int64_t groups) {
    if (headdim != mm::kSsdP || d_state != mm::kSsdN || batch <= 0 || !ssd_sizes_ok(batch, seqlen, heads, groups))
        return 0;
    return plan_ssd(batch, seqlen, heads).total;
}

mm_status mamba_ssd_fwd(const void* x, const void* z, const void* dt, const float* dt_bias, const float* A,
                        const void* Bm, const void* Cm, const float* Dskip, const float* h0,
                        void* y, float* h_last,
                        int64_t batch, int64_t seqlen, int64_t heads, int64_t headdim, int64_t d_state,
                        int64_t groups, void* workspace, size_t workspace_bytes, void* stream)
{
    if (!ssd_sizes_ok(batch, seqlen, heads, groups)) return MM_ERR_SHAPE;
    if (headdim != mm::kSsdP || d_state != mm::kSsdN) return MM_ERR_UNSUPPORTED;
    if (batch == 0) return MM_OK;
    const bool tokens = seqlen > 0;
    if (!A || !h_last || (tokens && (!x || !dt || !Bm || !Cm || !y))) return MM_ERR_NULL;
    for (const void* q : {x, z, dt, static_cast<const void*>(dt_bias), static_cast<const void*>(A), Bm, Cm,
                          static_cast<const void*>(Dskip), static_cast<const void*>(h0), static_cast<const void*>(y),
                          static_cast<const void*>(h_last)})
        if (q && !aligned16(q)) return MM_ERR_ALIGN;
    const int64_t C = heads * mm::kSsdP, NL = batch * seqlen;
    const Span sx = span(x, NL * C * 2), sz = span(z, NL * C * 2), sdt = span(dt, NL * heads * 2),
               sbias = span(dt_bias, heads * 4), sa = span(A, heads * 4), sb = span(Bm, NL * groups * mm::kSsdN * 2),
               sc = span(Cm, NL * groups * mm::kSsdN * 2), sd = span(Dskip, heads * 4),
               sh0 = span(h0, batch * C * mm::kSsdN * 4), sy = span(y, NL * C * 2),
               shl = span(h_last, batch * C * mm::kSsdN * 4);
    const Span ins[] = {sx, sz, sdt, sbias, sa, sb, sc, sd, sh0};
    for (const Span& in : ins)
        if (overlaps(sy, in) || overlaps(shl, in)) return MM_ERR_ALIAS;
    if (overlaps(sy, shl)) return MM_ERR_ALIAS;
    const SsdPlan pl = plan_ssd(batch, seqlen, heads);
    if (!workspace || workspace_bytes < pl.total) return MM_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MM_ERR_ALIGN;
    const Span sw = span(workspace, static_cast<int64_t>(pl.total));
    for (const Span& in : ins)
        if (overlaps(sw, in)) return MM_ERR_ALIAS;
    if (overlaps(sw, sy) || overlaps(sw, shl)) return MM_ERR_ALIAS;
    if (mm_status st = check_device(); st != MM_OK) return st;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned char* w = static_cast<unsigned char*>(workspace);
    unsigned long long* hdr = reinterpret_cast<unsigned long long*>(w);
    const unsigned long long epoch = next_call_id();   // written into hdr[1] by the state-passing launch
    mm::SsdParams p{};
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.z = static_cast<const __nv_bfloat16*>(z);
    p.dt = static_cast<const __nv_bfloat16*>(dt);
    p.dt_bias = dt_bias;
    p.A = A;
    p.Bm = static_cast<const __nv_bfloat16*>(Bm);
    p.Cm = static_cast<const __nv_bfloat16*>(Cm);
    p.Dskip = Dskip;
    p.h0 = h0;
    p.y = static_cast<__nv_bfloat16*>(y);
    p.h_last = h_last;
    p.S = reinterpret_cast<float*>(w + pl.off_s);
    p.Hin = reinterpret_cast<__nv_bfloat16*>(w + pl.off_hin);
    p.hin_lo = batch * pl.chunks * heads * mm::kSsdP * mm::kSsdN;
    p.dec = reinterpret_cast<float*>(w + pl.off_dec);
    p.L = seqlen;
    p.H = static_cast<int>(heads);
    p.G = static_cast<int>(groups);
    p.chunks = static_cast<int>(pl.chunks);
    p.batch = static_cast<int>(batch);
    p.wait_limit = copy_wait_limit();
    p.status = hdr;
    p.status_epoch = epoch;

    const dim3 cgrid(static_cast<unsigned>(pl.chunks), static_cast<unsigned>(heads), static_cast<unsigned>(batch));
    const bool fail = forced_launch_failure();
    CUtensorMap tc, tb, th, tx, tz, ty;
    if (pl.chunks > 0) {
        const int64_t gn = groups * mm::kSsdN;
        if (!encode_sw128_3d(&tc, Cm, gn, seqlen, batch, mm::kSsdQ) ||
            !encode_sw128_3d(&tb, Bm, gn, seqlen, batch, mm::kSsdQ) ||
            !encode_sw128_3d(&tx, x, C, seqlen, batch, mm::kSsdQ) ||
            !encode_sw128_3d(&tz, z ? z : x, C, seqlen, batch, mm::kSsdQ) ||
            !encode_sw128_3d(&ty, y, C, seqlen, batch, mm::kSsdQ) ||
            !encode_sw128_3d(&th, p.Hin, mm::kSsdN, 2 * batch * pl.chunks * heads * mm::kSsdP, 1, mm::kSsdP))
            return MM_ERR_CUDA;
        static std::atomic<unsigned long long> allowed_state{0};
        if (allow_smem(mm::ssd_chunk_state_kernel, allowed_state) != cudaSuccess) { cudaGetLastError(); return MM_ERR_CUDA; }
        mm::ssd_chunk_state_kernel<<<cgrid, mm::kSsdThreads,
                                     fail ? (1 << 20) : mm::SsdStateLayout::smem_bytes, s>>>(p, tb, tx);
        if (cudaGetLastError() != cudaSuccess) return MM_ERR_CUDA;
    }
    const int64_t quads = heads * mm::kSsdP * mm::kSsdN / 4;
    mm::ssd_state_pass_kernel<<<dim3(static_cast<unsigned>((quads + 255) / 256), static_cast<unsigned>(batch)), 256, 0,
                                s>>>(p);
    if (cudaGetLastError() != cudaSuccess) return MM_ERR_CUDA;
    if (pl.chunks > 0) {
        static std::atomic<unsigned long long> allowed_scan{0};
        if (allow_smem(mm::ssd_chunk_scan_kernel, allowed_scan) != cudaSuccess) { cudaGetLastError(); return MM_ERR_CUDA; }
        mm::ssd_chunk_scan_kernel<<<cgrid, mm::kSsdScanThreads,
                                    fail ? (1 << 20) : mm::SsdScanLayout::smem_bytes, s>>>(p, tc, tb, th, tx, tz, ty);
        if (cudaGetLastError() != cudaSuccess) return MM_ERR_CUDA;
    }
    return MM_OK;
}

mm_status mamba_ssd_state_update(const void* x, const void* z, const void* dt, const float* dt_bias,
                                 const float* A, const void* Bm, const void* Cm, const float* Dskip,
                                 float* state, void* y,
                                 int64_t batch, int64_t heads, int64_t headdim, int64_t d_state, int64_t groups,
                                 void* stream)
{
    if (batch < 0 || heads <= 0 || groups <= 0 || heads % groups != 0 || batch > 65535 || heads > (1 << 20))
        return MM_ERR_SHAPE;
    if (headdim != mm::kSsdP || d_state != mm::kSsdN) return MM_ERR_UNSUPPORTED;
    if (batch == 0) return MM_OK;
    if (!x || !dt || !A || !Bm || !Cm || !state || !y) return MM_ERR_NULL;
    for (const void* q : {x, z, dt, static_cast<const void*>(dt_bias), static_cast<const void*>(A), Bm, Cm,
                          static_cast<const void*>(Dskip), static_cast<const void*>(state), static_cast<const void*>(y)})
        if (q && !aligned16(q)) return MM_ERR_ALIGN;
    const int64_t C = heads * mm::kSsdP;
    const Span sx = span(x, batch * C * 2), sz = span(z, batch * C * 2), sdt = span(dt, batch * heads * 2),
               sbias = span(dt_bias, heads * 4), sa = span(A, heads * 4),
               sb = span(Bm, batch * groups * mm::kSsdN * 2), sc = span(Cm, batch * groups * mm::kSsdN * 2),
               sd = span(Dskip, heads * 4), sst = span(state, batch * C * mm::kSsdN * 4), sy = span(y, batch * C * 2);
    const Span ins[] = {sx, sz, sdt, sbias, sa, sb, sc, sd};
    for (const Span& in : ins)
        if (overlaps(sy, in) || overlaps(sst, in)) return MM_ERR_ALIAS;
    if (overlaps(sy, sst)) return MM_ERR_ALIAS;
    if (mm_status st = check_device(); st != MM_OK) return st;

    mm::SsdDecodeParams p{};
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.z = static_cast<const __nv_bfloat16*>(z);
    p.dt = static_cast<const __nv_bfloat16*>(dt);
    p.dt_bias = dt_bias;
    p.A = A;
    p.Bm = static_cast<const __nv_bfloat16*>(Bm);
    p.Cm = static_cast<const __nv_bfloat16*>(Cm);
    p.Dskip = Dskip;
    p.state = state;
    p.y = static_cast<__nv_bfloat16*>(y);
    p.H = static_cast<int>(heads);
    p.G = static_cast<int>(groups);
    mm::ssd_state_update_kernel<<<dim3(static_cast<unsigned>(heads), static_cast<unsigned>(batch)),
                                  mm::kSsdDecThreads, forced_launch_failure() ? (1 << 20) : 0,
                                  static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? MM_OK : MM_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------- Mamba-3 form (chunked fp32 recurrence)
namespace {

// Time chunks of mamba_m3_fwd: enough that the grid holds about 8 CTAs of
// 128 channels per SM, in whole 32-token tiles.  Workspace (256-byte
// aligned regions): header [256 B]; end states [K-1][B][H*P][16] fp32;
// chunk products [K-1][B][H][16] fp32.
struct M3Plan {
    int chunks = 1;
    int64_t chunk_len = 0;
    size_t off_state = 0, off_prod = 0, total = 0;
};

M3Plan plan_m3(int64_t batch, int64_t seqlen, int64_t heads, int sms) {
    M3Plan pl;
    const int64_t ctas = std::max<int64_t>(1, batch * heads * mm::kM3P / mm::kM3Threads);
    const int64_t want = std::min<int64_t>(64, std::max<int64_t>(1, (int64_t(sms) * 8 + ctas - 1) / ctas));
    const int64_t tiles = std::max<int64_t>(1, (seqlen + mm::kM3Tile - 1) / mm::kM3Tile);
    pl.chunk_len = ((tiles + want - 1) / want) * mm::kM3Tile;
    pl.chunks = static_cast<int>(seqlen > 0 ? (seqlen + pl.chunk_len - 1) / pl.chunk_len : 1);
    const size_t k1 = static_cast<size_t>(pl.chunks - 1), B = static_cast<size_t>(batch);
    pl.off_state = kWsHeader;
    pl.off_prod = pl.off_state + align256(k1 * B * heads * mm::kM3P * mm::kM3N * 4);
    pl.total = pl.off_prod + align256(k1 * B * heads * mm::kM3N * 4);
    return pl;
}

// The summary pass (when the sequence is cut in time) and the full pass, for
// R inputs per state.
template <int R>
cudaError_t launch_m3(const mm::M3Params& p, unsigned cx, int64_t batch, cudaStream_t s) {
    const int smem = forced_launch_failure() ? (1 << 20) : mm::m3_layout(R).bytes();
    static std::atomic<unsigned long long> allowed_sum{0}, allowed_full{0};
    cudaError_t e = allow_smem(mm::m3_chunk_kernel<false, R>, allowed_sum);
    if (e == cudaSuccess) e = allow_smem(mm::m3_chunk_kernel<true, R>, allowed_full);
    if (e != cudaSuccess) return e;
    if (p.chunks > 1) {
        mm::m3_chunk_kernel<false, R><<<dim3(cx, static_cast<unsigned>(p.chunks - 1), static_cast<unsigned>(batch)),
                                        mm::kM3Block, smem, s>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // The full pass is a programmatic dependent of the summary pass: its
    // chunk-0 CTAs run alongside the summary, the others wait for it in the
    // kernel before reading the summaries.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cx, static_cast<unsigned>(p.chunks), static_cast<unsigned>(batch));
    cfg.blockDim = dim3(mm::kM3Block);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.chunks > 1 ? 1 : 0;
    if ((e = cudaLaunchKernelEx(&cfg, mm::m3_chunk_kernel<true, R>, p)) != cudaSuccess) return e;
    return cudaGetLastError();
}

bool m3_sizes_ok(int64_t batch, int64_t seqlen, int64_t rank, int64_t heads, int64_t groups) {
    if (batch < 0 || seqlen < 0 || heads <= 0 || groups <= 0 || heads % groups != 0) return false;
    if (rank != 1 && rank != 2 && rank != 4) return false;
    if (heads % mm::kM3Heads != 0 || batch > 65535 || heads > (1 << 20)) return false;
    int64_t tokens;
    return mul_ok(batch, seqlen, &tokens) && tokens < (int64_t(1) << 40) / (rank * heads * mm::kM3P * 2);
}

}  // namespace

extern "C" {

size_t mamba_m3_workspace_size(int64_t batch, int64_t seqlen, int64_t rank, int64_t heads, int64_t headdim,
                               int64_t d_state, int64_t groups) {
    if (headdim != mm::kM3P || d_state != mm::kM3N || batch <= 0 || !m3_sizes_ok(batch, seqlen, rank, heads, groups))
        return 0;
    return plan_m3(batch, seqlen, heads, plan_sms()).total;
}

mm_status mamba_m3_fwd(const void* x, const void* z, const void* dt, const void* trap, const float* dt_bias,
                       const float* A, const float* theta, const void* Bm, const void* Cm, const float* Dskip,
                       const float* h0, const void* x_prev, const void* B_prev, void* y, float* h_last,
                       int64_t batch, int64_t seqlen, int64_t rank, int64_t heads, int64_t headdim,
                       int64_t d_state, int64_t groups, void* workspace, size_t workspace_bytes, void* stream)
{
    if (headdim != mm::kM3P || d_state != mm::kM3N) return MM_ERR_UNSUPPORTED;
    if (rank != 1 && rank != 2 && rank != 4) return MM_ERR_UNSUPPORTED;
    if (heads > 0 && heads % mm::kM3Heads != 0) return MM_ERR_UNSUPPORTED;
    if (!m3_sizes_ok(batch, seqlen, rank, heads, groups)) return MM_ERR_SHAPE;
    if (batch == 0) return MM_OK;
    const bool tokens = seqlen > 0;
    if (!A || !theta || !h_last || (tokens && (!x || !dt || !Bm || !Cm || !y))) return MM_ERR_NULL;
    if ((x_prev == nullptr) != (B_prev == nullptr)) return MM_ERR_NULL;
    for (const void* q : {x, z, dt, trap, static_cast<const void*>(dt_bias), static_cast<const void*>(A),
                          static_cast<const void*>(theta), Bm, Cm, static_cast<const void*>(Dskip),
                          static_cast<const void*>(h0), x_prev, B_prev, static_cast<const void*>(y),
                          static_cast<const void*>(h_last)})
        if (q && !aligned16(q)) return MM_ERR_ALIGN;
    const int64_t C = heads * mm::kM3P, NL = batch * seqlen;
    const int64_t bc = groups * mm::kM3N;
    const Span sx = span(x, NL * rank * C * 2), sz = span(z, NL * rank * C * 2), sdt = span(dt, NL * heads * 2),
               str = span(trap, NL * heads * 2), sbias = span(dt_bias, heads * 4), sa = span(A, heads * 4),
               sth = span(theta, heads * mm::kM3Pairs * 4), sb = span(Bm, NL * rank * bc * 2),
               sc = span(Cm, NL * rank * bc * 2), sd = span(Dskip, heads * 4),
               sh0 = span(h0, batch * C * mm::kM3N * 4), sxp = span(x_prev, batch * rank * C * 2),
               sbp = span(B_prev, batch * rank * bc * 2), sy = span(y, NL * rank * C * 2),
               shl = span(h_last, batch * C * mm::kM3N * 4);
    const Span ins[] = {sx, sz, sdt, str, sbias, sa, sth, sb, sc, sd, sh0, sxp, sbp};
    for (const Span& in : ins)
        if (overlaps(sy, in) || overlaps(shl, in)) return MM_ERR_ALIAS;
    if (overlaps(sy, shl)) return MM_ERR_ALIAS;
    const int sms = plan_sms();
    const M3Plan pl = plan_m3(batch, seqlen, heads, sms);
    if (!workspace || workspace_bytes < pl.total) return MM_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MM_ERR_ALIGN;
    const Span sw = span(workspace, static_cast<int64_t>(pl.total));
    for (const Span& in : ins)
        if (overlaps(sw, in)) return MM_ERR_ALIAS;
    if (overlaps(sw, sy) || overlaps(sw, shl)) return MM_ERR_ALIAS;
    if (mm_status st = check_device(); st != MM_OK) return st;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned char* w = static_cast<unsigned char*>(workspace);
    mm::M3Params p{};
    // the call's status word: the full pass writes the epoch into the
    // header's second word (these kernels have no wait that can give up, so
    // the status always reads complete)
    p.status = reinterpret_cast<unsigned long long*>(w);
    p.status_epoch = next_call_id();
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.z = static_cast<const __nv_bfloat16*>(z);
    p.dt = static_cast<const __nv_bfloat16*>(dt);
    p.trap = static_cast<const __nv_bfloat16*>(trap);
    p.dt_bias = dt_bias;
    p.A = A;
    p.theta = theta;
    p.Bm = static_cast<const __nv_bfloat16*>(Bm);
    p.Cm = static_cast<const __nv_bfloat16*>(Cm);
    p.Dskip = Dskip;
    p.h0 = h0;
    p.x_prev = static_cast<const __nv_bfloat16*>(x_prev);
    p.B_prev = static_cast<const __nv_bfloat16*>(B_prev);
    p.y = static_cast<__nv_bfloat16*>(y);
    p.h_last = h_last;
    p.ws_state = reinterpret_cast<float*>(w + pl.off_state);
    p.ws_prod = reinterpret_cast<float*>(w + pl.off_prod);
    p.L = seqlen;
    p.chunk_len = pl.chunk_len;
    p.R = static_cast<int>(rank);
    p.H = static_cast<int>(heads);
    p.G = static_cast<int>(groups);
    p.chunks = pl.chunks;
    const unsigned cx = static_cast<unsigned>(C / mm::kM3Threads);
    cudaError_t e = rank == 1 ? launch_m3<1>(p, cx, batch, s) : rank == 2 ? launch_m3<2>(p, cx, batch, s)
                                                                          : launch_m3<4>(p, cx, batch, s);
    if (e != cudaSuccess) { cudaGetLastError(); return MM_ERR_CUDA; }
    return MM_OK;
}

mm_status mamba_m3_state_update(const void* x, const void* z, const void* dt, const void* trap, const float* dt_bias,
                                const float* A, const float* theta, const void* Bm, const void* Cm,
                                const float* Dskip, float* state, const void* x_prev, const void* B_prev, void* y,
                                int64_t batch, int64_t rank, int64_t heads, int64_t headdim, int64_t d_state,
                                int64_t groups, void* stream)
{
    if (headdim != mm::kM3P || d_state != mm::kM3N) return MM_ERR_UNSUPPORTED;
    if (rank != 1 && rank != 2 && rank != 4) return MM_ERR_UNSUPPORTED;
    if (heads > 0 && heads % mm::kM3Heads != 0) return MM_ERR_UNSUPPORTED;
    if (!m3_sizes_ok(batch, 1, rank, heads, groups)) return MM_ERR_SHAPE;
    if (batch == 0) return MM_OK;
    if (!x || !dt || !A || !theta || !Bm || !Cm || !state || !y) return MM_ERR_NULL;
    if ((x_prev == nullptr) != (B_prev == nullptr)) return MM_ERR_NULL;
    for (const void* q : {x, z, dt, trap, static_cast<const void*>(dt_bias), static_cast<const void*>(A),
                          static_cast<const void*>(theta), Bm, Cm, static_cast<const void*>(Dskip),
                          static_cast<const void*>(state), x_prev, B_prev, static_cast<const void*>(y)})
        if (q && !aligned16(q)) return MM_ERR_ALIGN;
    const int64_t C = heads * mm::kM3P;
    const int64_t bc = groups * mm::kM3N;
    const Span sx = span(x, batch * rank * C * 2), sz = span(z, batch * rank * C * 2),
               sdt = span(dt, batch * heads * 2), str = span(trap, batch * heads * 2),
               sbias = span(dt_bias, heads * 4), sa = span(A, heads * 4), sth = span(theta, heads * mm::kM3Pairs * 4),
               sb = span(Bm, batch * rank * bc * 2), sc = span(Cm, batch * rank * bc * 2), sd = span(Dskip, heads * 4),
               sxp = span(x_prev, batch * rank * C * 2), sbp = span(B_prev, batch * rank * bc * 2),
               sst = span(state, batch * C * mm::kM3N * 4), sy = span(y, batch * rank * C * 2);
    const Span ins[] = {sx, sz, sdt, str, sbias, sa, sth, sb, sc, sd, sxp, sbp};
    for (const Span& in : ins)
        if (overlaps(sy, in) || overlaps(sst, in)) return MM_ERR_ALIAS;
    if (overlaps(sy, sst)) return MM_ERR_ALIAS;
    if (mm_status st = check_device(); st != MM_OK) return st;

    mm::M3DecodeParams p{};
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.z = static_cast<const __nv_bfloat16*>(z);
    p.dt = static_cast<const __nv_bfloat16*>(dt);
    p.trap = static_cast<const __nv_bfloat16*>(trap);
    p.dt_bias = dt_bias;
    p.A = A;
    p.theta = theta;
    p.Bm = static_cast<const __nv_bfloat16*>(Bm);
    p.Cm = static_cast<const __nv_bfloat16*>(Cm);
    p.Dskip = Dskip;
    p.state = state;
    p.x_prev = static_cast<const __nv_bfloat16*>(x_prev);
    p.B_prev = static_cast<const __nv_bfloat16*>(B_prev);
    p.y = static_cast<__nv_bfloat16*>(y);
    p.H = static_cast<int>(heads);
    p.G = static_cast<int>(groups);
    const dim3 grid(static_cast<unsigned>(heads / mm::kM3Heads), static_cast<unsigned>(batch));
    const size_t smem = forced_launch_failure() ? (size_t(1) << 20) : 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (rank == 1) mm::m3_state_update_kernel<1><<<grid, mm::kM3DecThreads, smem, s>>>(p);
    else if (rank == 2) mm::m3_state_update_kernel<2><<<grid, mm::kM3DecThreads, smem, s>>>(p);
    else mm::m3_state_update_kernel<4><<<grid, mm::kM3DecThreads, smem, s>>>(p);
    return cudaGetLastError() == cudaSuccess ? MM_OK : MM_ERR_CUDA;
}

}  // extern "C"
