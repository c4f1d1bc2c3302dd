// la2_api.cu -- the C ABI of libla2.so (declared in include/la2.h): argument
// validation, TMA descriptor set-up and kernel launch.  Everything numerical
// happens in the kernels of scan_ws_sm100.cuh (bf16 inputs) and scan_f32.cuh
// (fp32 inputs).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>
#include <atomic>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "decode.cuh"
#include "dlambda.cuh"
#include "la2.h"
#include "normalize.cuh"
#include "scan_blk_sm100.cuh"
#include "scan_f32.cuh"
#include "scan_ws_sm100.cuh"

namespace {

__device__ int g_la2_status = 0;  // device status word (see la2_device_status)
__device__ int g_la2_never_set = 0;  // la2_selftest_timeout's flag: nothing ever writes it

thread_local int t_last_launches = 0;

constexpr int kMaxDevices = 64;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

template <int DA, int DC, bool kNorm = false>
bool set_ws_attrs() {
    constexpr size_t smem = la2::ws::Smem<DA, DC, kNorm>::kBytes;
    if constexpr (!kNorm) {  // the bf16-output instantiations (no normalised form)
        if (cudaFuncSetAttribute(la2::ws::la2_scan_ws<DA, DC, false, false, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
            cudaFuncSetAttribute(la2::ws::la2_scan_ws<DA, DC, true, false, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return false;
    }
    return cudaFuncSetAttribute(la2::ws::la2_scan_ws<DA, DC, false, kNorm>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess &&
           cudaFuncSetAttribute(la2::ws::la2_scan_ws<DA, DC, true, kNorm>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess &&
           cudaFuncSetAttribute(la2::ws::la2_state_ws<DA, DC>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                la2::ws::StateSmem<DA, DC>::kBytes) == cudaSuccess;
}

template <int DA, int TB>
bool set_blk_attrs() {
    return cudaFuncSetAttribute(la2::blk::la2_scan_blk<DA, TB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                la2::blk::Smem<DA, TB>::kBytes) == cudaSuccess;
}

// How the bf16 kernel spreads its (sequence, role) units over CTAs.  Each CTA
// fills one SM (148 on a B200).  Two plans:
//
// - uniform: each unit is cut into g equal segments, one CTA each; g > 1
//   only when there are fewer units than SMs;
// - balanced: the units' tiles are laid end to end and CTA c takes tiles
//   [c L, (c+1) L), L = ceil(total / 148): one wave, every SM the same work, a
//   CTA running the end of one unit and the start of the next one after the
//   other.
// The default (AUTO, auto_balanced below) takes balanced only where the
// uniform waves leave a mostly empty last wave over long units.
//
// A segment that does not start its unit gets its incoming state from the
// state pre-pass, which reads that unit's B and C up to the segment.  Filling
// more SMs does not always pay: a tile takes 20-40% longer once every SM runs
// the scan (at d = 128 the scan then nears what the memory system delivers), a
// partial last wave runs faster, and the pre-pass re-reads B and C.
//
// Workspace, flat in T in both plans: uniform, (g - 1) states per unit with g
// from the number of units alone (a short sequence may use fewer); balanced,
// one state per CTA boundary, at most 147.
constexpr int kTargetCTAs = 148;
constexpr int kMaxSegments = 32;

std::atomic<int> g_schedule{LA2_SCHEDULE_AUTO};

int max_segments(long long units) {
    if (units <= 0 || units >= kTargetCTAs) return 1;
    const long long g = kTargetCTAs / units;
    return static_cast<int>(g < kMaxSegments ? g : kMaxSegments);
}

struct SegPlan {
    int balanced = 0;
    int nseg = 1;        // uniform: segments per unit
    int seg_tiles = 1;   // L
    long long nctas = 0, npre = 0;  // scan and pre-pass grids
};

long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

SegPlan uniform_plan(long long units, int nb) {
    int g = max_segments(units);
    const int cap = nb / 2 > 1 ? nb / 2 : 1;
    if (g > cap) g = cap;
    SegPlan sp;
    sp.seg_tiles = static_cast<int>(cdiv(nb, g));
    sp.nseg = static_cast<int>(cdiv(nb, sp.seg_tiles));
    sp.nctas = units * sp.nseg;
    sp.npre = units * (sp.nseg - 1);
    return sp;
}

// Returns false when the balanced plan does not apply (segment length out of
// the kernel's int range).
bool balanced_plan(long long units, int nb, SegPlan* out) {
    const long long total = units * nb;
    const long long L = cdiv(total, kTargetCTAs);
    if (L < 1 || L > (1LL << 28)) return false;
    SegPlan sp;
    sp.balanced = 1;
    sp.seg_tiles = static_cast<int>(L);
    sp.nctas = cdiv(total, L);
    sp.npre = L % nb != 0 ? sp.nctas - 1 : 0;  // some CTA boundary falls inside a unit
    *out = sp;
    return true;
}

// AUTO takes the balanced plan where the uniform one runs its units in waves
// whose last is mostly empty (at least 148 units, over a quarter of the
// waves' SM time idle) and the units are long (>= 128 tiles), so that one
// balanced wave saves more than its state pre-pass costs; elsewhere the
// uniform plan.  bench.py on B200, processes alternating the schedules
// (tokens/s, uniform -> balanced):
//   T =  65,536, 2 x 32 sequences (bwd: 192 units, second wave 44 CTAs): 19.2 -> 20.2 M
//   T = 131,072, 32 sequences (fwd in 4 segments, bwd 96 units): 19.4 -> 19.2 M
//   long, 16 sequences of 65,536 (fwd in 9 segments, bwd in 3):      38.6 -> 37.8 M
bool auto_balanced(long long units, int nb) {
    if (units < kTargetCTAs || nb < 128) return false;
    const long long waves = cdiv(units, kTargetCTAs);
    return 4 * units < 3 * kTargetCTAs * waves;
}

// `sched` is the schedule setting read once at the top of the entry point, so
// that one call sizes its workspace and launches with the same plan even if
// another thread changes the setting meanwhile.
SegPlan plan_segments(long long units, int T, int sched) {
    const int nb = (T + la2::ws::kTB - 1) / la2::ws::kTB;
    SegPlan b;
    const bool bal = sched == LA2_SCHEDULE_BALANCED || (sched == LA2_SCHEDULE_AUTO && auto_balanced(units, nb));
    if (bal && balanced_plan(units, nb, &b)) return b;
    return uniform_plan(units, nb);
}

// Workspace bytes of one bf16 launch over `units` (sequence, role) units,
// the same for every T: the balanced plan's 147 states (never fewer than the
// uniform plan's states at the segment boundaries of every unit), or the
// uniform plan's.  AUTO reserves the balanced size for unit counts it takes
// the balanced plan for at some T (the set of such T, if any, contains every
// long T, so the test at a very long T decides).
size_t seg_workspace_bytes(long long units, int da, int dc, int sched) {
    const size_t state = static_cast<size_t>(da) * static_cast<size_t>(dc) * sizeof(float);
    const bool bal = sched == LA2_SCHEDULE_BALANCED || (sched == LA2_SCHEDULE_AUTO && auto_balanced(units, 1 << 20));
    if (bal) return static_cast<size_t>(kTargetCTAs - 1) * state;
    return static_cast<size_t>(max_segments(units) - 1) * static_cast<size_t>(units) * state;
}

// The gradient in lambda (dlambda.cuh): each sequence is cut into g segments
// of a multiple of 32 rows, g = min(32, 148 / sequences) (at least 1), so that
// few sequences still fill the SMs.  Workspace, flat in T: one fp64 partial
// sum per (sequence, segment) and the fp32 (W, U) pair at the end of every
// segment but the last.
struct DlPlan {
    int g = 1;         // segments the workspace is sized for
    int nseg = 1;      // segments of this T (<= g)
    int seg_rows = 0;  // rows per segment
};

DlPlan dl_plan(long long seqs, int T) {
    DlPlan pl;
    pl.g = static_cast<int>(seqs >= kTargetCTAs ? 1 : (kTargetCTAs / seqs < kMaxSegments ? kTargetCTAs / seqs
                                                                                          : kMaxSegments));
    if (pl.g < 1) pl.g = 1;
    const long long per = cdiv(T > 0 ? T : 1, pl.g);
    pl.seg_rows = static_cast<int>(cdiv(per, la2::kDlRows) * la2::kDlRows);
    pl.nseg = static_cast<int>(cdiv(T > 0 ? T : 1, pl.seg_rows));
    return pl;
}

size_t dl_workspace_bytes(long long seqs, int T, int d, int e) {
    const DlPlan pl = dl_plan(seqs, T);
    size_t partial = static_cast<size_t>(seqs) * pl.g * sizeof(double);
    partial = (partial + 255) & ~static_cast<size_t>(255);
    return partial + static_cast<size_t>(seqs) * (pl.g - 1) * 2 * d * e * sizeof(float);
}

// The normalised form (normalize.cuh): each sequence is cut into chunks of a
// multiple of 32 rows, g = min(64, ceil(8 * 148 / sequences)) (at least 1), the
// 128-thread scans then filling the SMs several CTAs deep.  Chunk end states
// (one d-vector each but the last) sit in the workspace, flat in T.
struct NzPlan {
    int g = 1, nchunk = 1, rows = 0;
};

NzPlan nz_plan(long long seqs, int T) {
    NzPlan pl;
    const long long want = cdiv(8LL * kTargetCTAs, seqs > 0 ? seqs : 1);
    pl.g = static_cast<int>(want < 1 ? 1 : (want > 64 ? 64 : want));
    const long long per = cdiv(T > 0 ? T : 1, pl.g);
    pl.rows = static_cast<int>(cdiv(per, la2::kNzRows) * la2::kNzRows);
    pl.nchunk = static_cast<int>(cdiv(T > 0 ? T : 1, pl.rows));
    return pl;
}

size_t nz_chunk_bytes(long long seqs, int T, int d) {
    const NzPlan pl = nz_plan(seqs, T);
    return static_cast<size_t>(seqs) * (pl.g - 1) * d * sizeof(float);
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct DeviceState {
    std::once_flag once;
    int* status = nullptr;
    int* never_set = nullptr;
    bool ok = false;
};
DeviceState g_dev[kMaxDevices];

// Per-device set-up: address of the status word, dynamic shared-memory limits.
bool device_setup(int* dev_out, int** status_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
    DeviceState& s = g_dev[dev];
    std::call_once(s.once, [&s] {
        void* p = nullptr;
        bool ok = cudaGetSymbolAddress(&p, g_la2_status) == cudaSuccess;
        s.status = static_cast<int*>(p);
        void* f = nullptr;
        ok = ok && cudaGetSymbolAddress(&f, g_la2_never_set) == cudaSuccess;
        s.never_set = static_cast<int*>(f);
        ok = ok && set_ws_attrs<64, 64>() && set_ws_attrs<64, 128>() && set_ws_attrs<128, 64>() &&
             set_ws_attrs<128, 128>() && set_ws_attrs<64, 64, true>() && set_ws_attrs<64, 128, true>() &&
             set_ws_attrs<128, 64, true>() && set_ws_attrs<128, 128, true>();
        ok = ok && set_blk_attrs<64, 64>() && set_blk_attrs<64, 256>() && set_blk_attrs<128, 64>() &&
             set_blk_attrs<128, 256>();
        ok = ok &&
             cudaFuncSetAttribute(la2::la2_dlam_scan<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(la2::dl_scan_smem_bytes())) == cudaSuccess &&
             cudaFuncSetAttribute(la2::la2_dlam_scan<__nv_bfloat16>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(la2::dl_scan_smem_bytes())) == cudaSuccess;
        ok = ok && cudaFuncSetAttribute(la2::la2_scan_f32,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(la2::f32_scan_smem_bytes(128, 128, 256))) ==
                       cudaSuccess;
        s.ok = ok;
    });
    if (!s.ok) return false;
    *dev_out = dev;
    *status_out = s.status;
    return true;
}

int* never_set_flag() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    return g_dev[dev].ok ? g_dev[dev].never_set : nullptr;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 4-D tensor map over a contiguous bf16 tensor [B, H, T, D] (dims D, T, H, B)
// or, with bthd, [B, T, H, D] (dims D, H, T, B), with strides increasing in
// both cases.  Box: 64 columns (128 bytes) x 128 positions of one (b, h),
// 128-byte swizzle; positions past T read as zero.
bool make_map(CUtensorMap* m, const void* ptr, int B, int H, int T, int D, bool bthd) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t esz = 2;
    const cuuint64_t d = static_cast<cuuint64_t>(D), t = static_cast<cuuint64_t>(T);
    const cuuint64_t h = static_cast<cuuint64_t>(H), b = static_cast<cuuint64_t>(B);
    const cuuint64_t dims[4] = {d, bthd ? h : t, bthd ? t : h, b};
    const cuuint64_t strides[3] = {d * esz, (bthd ? h : t) * d * esz, t * h * d * esz};
    const cuuint32_t box[4] = {64, bthd ? 1u : static_cast<cuuint32_t>(la2::ws::kTB),
                               bthd ? static_cast<cuuint32_t>(la2::ws::kTB) : 1u, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct RoleDesc {
    const void* a;
    const void* b;
    const void* c;
    void* x;
    int da, dc, dir;
    const float* init = nullptr;  // state the scan starts from (see la2::ws::Role)
    float* fin = nullptr;         // state the scan ends with
    int init_t = 0;               // init stored transposed ([DC][DA])
    const float* colf = nullptr;  // per-position factor on the summed index ([B*H, T])
};

// Self-test only (la2_selftest_timeout): a device flag that nothing sets, which
// the scan kernel's producer waits on, bounded by `ns`, before its first load.
struct Hold {
    const int* flag = nullptr;
    unsigned long long ns = 0;
};

la2_status common_checks(int B, int H, int T, int d, int e, int block, la2_dtype dtype,
                         bool* empty) {
    if (dtype != LA2_DTYPE_F32 && dtype != LA2_DTYPE_BF16) return LA2_ERR_INVALID_ARG;
    if (block != 64 && block != 128 && block != 256) return LA2_ERR_INVALID_ARG;
    if (B < 0 || H < 0 || T < 0 || d <= 0 || e <= 0) return LA2_ERR_INVALID_ARG;
    *empty = (B == 0 || H == 0 || T == 0);
    if (*empty) return LA2_OK;
    if (static_cast<long long>(B) * H > (1LL << 24)) return LA2_ERR_UNSUPPORTED;
    if (dtype == LA2_DTYPE_BF16) {
        if ((d != 64 && d != 128) || (e != 64 && e != 128)) return LA2_ERR_UNSUPPORTED;
    } else {
        if (d > 128 || e > 128) return LA2_ERR_UNSUPPORTED;
    }
    return LA2_OK;
}

template <int DA, int DC, bool kNorm = false, bool kXb16 = false>
void launch_ws(const la2::ws::Params& p, const SegPlan& sp, cudaStream_t stream) {
    constexpr size_t smem = la2::ws::Smem<DA, DC, kNorm>::kBytes;
    if (sp.npre > 0)
        la2::ws::la2_state_ws<DA, DC><<<static_cast<unsigned>(sp.npre), la2::ws::kStateThreads,
                                        la2::ws::StateSmem<DA, DC>::kBytes, stream>>>(p);
    if (sp.balanced)
        la2::ws::la2_scan_ws<DA, DC, true, kNorm, kXb16>
            <<<static_cast<unsigned>(sp.nctas), la2::ws::kThreads, smem, stream>>>(p);
    else
        la2::ws::la2_scan_ws<DA, DC, false, kNorm, kXb16>
            <<<static_cast<unsigned>(sp.nctas), la2::ws::kThreads, smem, stream>>>(p);
}

// Launches the warp-specialised kernel over `n` roles that share (DA, DC),
// with the CTAs of plan_segments, preceded by the state pre-pass when some
// segment starts inside its unit.
la2_status launch_bf16_ws(const RoleDesc* roles, int n, const float* decay, int B, int H, int T,
                          bool bthd, int sched, int* status, float* seg_state, const Hold& hold,
                          cudaStream_t stream, bool norm = false, bool xbf16 = false) {
    la2::ws::Params p;
    std::memset(&p, 0, sizeof(p));
    const int BH = B * H;
    const int da = roles[0].da, dc = roles[0].dc;
    for (int r = 0; r < n; ++r) {
        if (!make_map(&p.role[r].ta, roles[r].a, B, H, T, da, bthd) ||
            !make_map(&p.role[r].tb, roles[r].b, B, H, T, da, bthd) ||
            !make_map(&p.role[r].tc, roles[r].c, B, H, T, dc, bthd))
            return LA2_ERR_CUDA;
        p.role[r].x = roles[r].x;
        p.role[r].init = roles[r].init;
        p.role[r].fin = roles[r].fin;
        p.role[r].dir = roles[r].dir;
        p.role[r].init_t = roles[r].init_t;
        p.role[r].colf = roles[r].colf;
    }
    p.decay = decay;
    p.status = status;
    p.H = H;
    p.T = T;
    p.nroles = n;
    p.bthd = bthd ? 1 : 0;
    p.hold = hold.flag;
    p.hold_ns = hold.ns;
    const SegPlan sp = plan_segments(static_cast<long long>(BH) * n, T, sched);
    p.nunits = BH * n;
    p.nseg = sp.nseg;
    p.seg_tiles = sp.seg_tiles;
    p.balanced = sp.balanced;
    p.seg_state = seg_state;
    if (sp.npre > 0 && !seg_state) return LA2_ERR_WORKSPACE;
    if (sp.nctas > 0x7fffffffLL) return LA2_ERR_UNSUPPORTED;
    if (norm) {
        if (da == 128 && dc == 128) launch_ws<128, 128, true>(p, sp, stream);
        else if (da == 128) launch_ws<128, 64, true>(p, sp, stream);
        else if (dc == 128) launch_ws<64, 128, true>(p, sp, stream);
        else launch_ws<64, 64, true>(p, sp, stream);
    } else if (xbf16) {
        if (da == 128 && dc == 128) launch_ws<128, 128, false, true>(p, sp, stream);
        else if (da == 128) launch_ws<128, 64, false, true>(p, sp, stream);
        else if (dc == 128) launch_ws<64, 128, false, true>(p, sp, stream);
        else launch_ws<64, 64, false, true>(p, sp, stream);
    } else {
        if (da == 128 && dc == 128) launch_ws<128, 128>(p, sp, stream);
        else if (da == 128) launch_ws<128, 64>(p, sp, stream);
        else if (dc == 128) launch_ws<64, 128>(p, sp, stream);
        else launch_ws<64, 64>(p, sp, stream);
    }
    if (cudaGetLastError() != cudaSuccess) return LA2_ERR_CUDA;
    t_last_launches += sp.npre > 0 ? 2 : 1;
    return LA2_OK;
}

// T_B = 64 or 256 on bf16 inputs (scan_blk_sm100.cuh): one CTA per
// (sequence, role, 64 value columns), no segments, no workspace; carried
// states and the per-position factor (colf) as in the T_B = 128 kernel.
la2_status launch_bf16_blk(const RoleDesc* roles, int n, const float* decay, int B, int H, int T,
                           int block, bool bthd, int* status, cudaStream_t stream, bool xbf16) {
    la2::blk::Params p;
    std::memset(&p, 0, sizeof(p));
    const int da = roles[0].da, dc = roles[0].dc;
    for (int r = 0; r < n; ++r) {
        if (!make_map(&p.role[r].ta, roles[r].a, B, H, T, da, bthd) ||
            !make_map(&p.role[r].tb, roles[r].b, B, H, T, da, bthd) ||
            !make_map(&p.role[r].tc, roles[r].c, B, H, T, dc, bthd))
            return LA2_ERR_CUDA;
        p.role[r].x = roles[r].x;
        p.role[r].dir = roles[r].dir;
        p.role[r].init = roles[r].init;
        p.role[r].fin = roles[r].fin;
        p.role[r].init_t = roles[r].init_t;
        p.role[r].colf = roles[r].colf;
    }
    p.decay = decay;
    p.status = status;
    p.H = H;
    p.T = T;
    p.nroles = n;
    p.bthd = bthd ? 1 : 0;
    p.dc = dc;
    p.nslice = dc / la2::blk::kDC;
    p.xbf16 = xbf16 ? 1 : 0;
    const long long ctas = static_cast<long long>(B) * H * n * p.nslice;
    if (ctas > 0x7fffffffLL) return LA2_ERR_UNSUPPORTED;
    const unsigned grid = static_cast<unsigned>(ctas);
    auto go = [&](auto kernel, size_t smem) {
        kernel<<<grid, la2::blk::kThreads, smem, stream>>>(p);
    };
    if (da == 128 && block == 256) go(la2::blk::la2_scan_blk<128, 256>, la2::blk::Smem<128, 256>::kBytes);
    else if (da == 128) go(la2::blk::la2_scan_blk<128, 64>, la2::blk::Smem<128, 64>::kBytes);
    else if (block == 256) go(la2::blk::la2_scan_blk<64, 256>, la2::blk::Smem<64, 256>::kBytes);
    else go(la2::blk::la2_scan_blk<64, 64>, la2::blk::Smem<64, 64>::kBytes);
    if (cudaGetLastError() != cudaSuccess) return LA2_ERR_CUDA;
    ++t_last_launches;
    return LA2_OK;
}

la2_status launch_f32(const RoleDesc* roles, int n, const float* decay, int B, int H, int T,
                      int block, bool bthd, cudaStream_t stream) {
    la2::F32Params p;
    std::memset(&p, 0, sizeof(p));
    int da_max = 0, dc_max = 0;
    for (int r = 0; r < n; ++r) {
        p.role[r].a = static_cast<const float*>(roles[r].a);
        p.role[r].b = static_cast<const float*>(roles[r].b);
        p.role[r].c = static_cast<const float*>(roles[r].c);
        p.role[r].x = static_cast<float*>(roles[r].x);
        p.role[r].da = roles[r].da;
        p.role[r].dc = roles[r].dc;
        p.role[r].dir = roles[r].dir;
        p.role[r].init = roles[r].init;
        p.role[r].fin = roles[r].fin;
        p.role[r].init_t = roles[r].init_t;
        p.role[r].colf = roles[r].colf;
        da_max = roles[r].da > da_max ? roles[r].da : da_max;
        dc_max = roles[r].dc > dc_max ? roles[r].dc : dc_max;
    }
    p.decay = decay;
    p.H = H;
    p.T = T;
    p.TB = block;
    p.nroles = n;
    p.bthd = bthd ? 1 : 0;
    const size_t smem = la2::f32_scan_smem_bytes(da_max, dc_max, block);
    const dim3 grid(static_cast<unsigned>(B * H * n));
    la2::la2_scan_f32<<<grid, la2::kF32Threads, smem, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return LA2_ERR_CUDA;
    ++t_last_launches;
    return LA2_OK;
}

// Groups roles with identical (DA, DC); each group is one launch (two with the
// state pre-pass).  Calls `f(group, m)` per group, in a fixed order.
template <class F>
la2_status for_role_groups(const RoleDesc* roles, int n, F&& f) {
    RoleDesc group[3];
    bool done[3] = {false, false, false};
    for (int r = 0; r < n; ++r) {
        if (done[r]) continue;
        int m = 0;
        for (int s = r; s < n; ++s)
            if (!done[s] && roles[s].da == roles[r].da && roles[s].dc == roles[r].dc) {
                group[m++] = roles[s];
                done[s] = true;
            }
        const la2_status st = f(group, m);
        if (st != LA2_OK) return st;
    }
    return LA2_OK;
}

size_t bf16_workspace_bytes(const RoleDesc* roles, int n, int B, int H, int T, int sched,
                            int block = la2::ws::kTB) {
    if (block != la2::ws::kTB) return 0;  // the T_B = 64 / 256 kernel needs none
    size_t total = 0;
    for_role_groups(roles, n, [&](const RoleDesc* g, int m) {
        total += seg_workspace_bytes(static_cast<long long>(B) * H * m, g[0].da, g[0].dc, sched);
        total = (total + 255) & ~static_cast<size_t>(255);
        return LA2_OK;
    });
    return total;
}

la2_status run_roles(const RoleDesc* roles, int n, const float* decay, int B, int H, int T,
                     int block, la2_dtype dtype, bool bthd, int sched, void* workspace,
                     size_t ws_bytes, cudaStream_t stream, const Hold& hold = Hold(),
                     bool norm = false, bool xbf16 = false) {
    int dev = 0;
    int* status = nullptr;
    if (dtype == LA2_DTYPE_BF16) {
        const size_t need = bf16_workspace_bytes(roles, n, B, H, T, sched, block);
        if (need > 0 && (workspace == nullptr || ws_bytes < need)) return LA2_ERR_WORKSPACE;
    }
    if (!device_setup(&dev, &status)) return LA2_ERR_CUDA;
    if (dtype == LA2_DTYPE_F32) {
        if (xbf16) return LA2_ERR_UNSUPPORTED;
        return launch_f32(roles, n, decay, B, H, T, block, bthd, stream);
    }
    if (block != la2::ws::kTB) {
        if (hold.flag) return LA2_ERR_UNSUPPORTED;  // the self-test runs the T_B = 128 kernel
        return for_role_groups(roles, n, [&](const RoleDesc* g, int m) {
            return launch_bf16_blk(g, m, decay, B, H, T, block, bthd, status, stream, xbf16);
        });
    }
    size_t off = 0;
    return for_role_groups(roles, n, [&](const RoleDesc* g, int m) {
        float* seg = workspace ? reinterpret_cast<float*>(static_cast<char*>(workspace) + off) : nullptr;
        off += seg_workspace_bytes(static_cast<long long>(B) * H * m, g[0].da, g[0].dc, sched);
        off = (off + 255) & ~static_cast<size_t>(255);
        return launch_bf16_ws(g, m, decay, B, H, T, bthd, sched, status, seg, hold, stream, norm,
                              xbf16);
    });
}


template <typename Tin>
void nz_launch(const la2::NzParams& p, long long seqs, cudaStream_t cs, int* launches) {
    if (p.nchunk > 1) {
        la2::la2_nz_prepass<Tin><<<static_cast<unsigned>(seqs * (p.nchunk - 1)), la2::kNzThreads, 0, cs>>>(p);
        ++*launches;
    }
    la2::la2_nz_scan<Tin><<<static_cast<unsigned>(seqs * p.nchunk), la2::kNzThreads, 0, cs>>>(p);
    ++*launches;
}

la2::NzParams nz_params(int B, int H, int T, int d, int e, bool bthd, const float* decay, float* chunk) {
    la2::NzParams p;
    std::memset(&p, 0, sizeof(p));
    const NzPlan pl = nz_plan(static_cast<long long>(B) * H, T);
    p.decay = decay;
    p.chunk = chunk;
    p.B = B;
    p.H = H;
    p.T = T;
    p.d = d;
    p.e = e;
    p.bthd = bthd ? 1 : 0;
    p.nchunk = pl.nchunk;
    p.chunk_rows = pl.rows;
    return p;
}

la2_status norm_checks(const void* q, const void* k, const void* v, const float* decay, int B, int H,
                       int T, int d, int e, int block, la2_dtype dtype, la2_layout layout, bool* empty) {
    if (layout != LA2_LAYOUT_BHTD && layout != LA2_LAYOUT_BTHD) return LA2_ERR_INVALID_ARG;
    const la2_status st = common_checks(B, H, T, d, e, block, dtype, empty);
    if (st != LA2_OK || *empty) return st;
    if (d > 128) return LA2_ERR_UNSUPPORTED;
    if (!q || !k || !v || !decay) return LA2_ERR_INVALID_ARG;
    return LA2_OK;
}

}  // namespace

extern "C" {

size_t la2_workspace_bytes(int B, int H, int T, int d, int e, int block, la2_dtype dtype,
                           int is_bwd) {
    bool empty = false;
    const la2_status st = common_checks(B, H, T, d, e, block, dtype, &empty);
    if (st != LA2_OK) return static_cast<size_t>(-1);
    if (empty || dtype != LA2_DTYPE_BF16) return 0;
    const RoleDesc fwd[1] = {{nullptr, nullptr, nullptr, nullptr, d, e, +1}};
    const RoleDesc bwd[3] = {{nullptr, nullptr, nullptr, nullptr, e, d, +1},
                             {nullptr, nullptr, nullptr, nullptr, e, d, -1},
                             {nullptr, nullptr, nullptr, nullptr, d, e, -1}};
    const int sched = g_schedule.load();
    return is_bwd ? bf16_workspace_bytes(bwd, 3, B, H, T, sched, block)
                  : bf16_workspace_bytes(fwd, 1, B, H, T, sched, block);
}

la2_schedule la2_set_schedule(la2_schedule schedule) {
    if (schedule != LA2_SCHEDULE_AUTO && schedule != LA2_SCHEDULE_UNIFORM &&
        schedule != LA2_SCHEDULE_BALANCED)
        return static_cast<la2_schedule>(g_schedule.load());
    return static_cast<la2_schedule>(g_schedule.exchange(schedule));
}

int la2_plan_info(int B, int H, int T, int d, int e, int block, la2_dtype dtype, int is_bwd,
                  la2_plan* out, int max_out) {
    bool empty = false;
    if (common_checks(B, H, T, d, e, block, dtype, &empty) != LA2_OK) return -1;
    if (empty || dtype != LA2_DTYPE_BF16) return 0;
    const RoleDesc fwd[1] = {{nullptr, nullptr, nullptr, nullptr, d, e, +1}};
    const RoleDesc bwd[3] = {{nullptr, nullptr, nullptr, nullptr, e, d, +1},
                             {nullptr, nullptr, nullptr, nullptr, e, d, -1},
                             {nullptr, nullptr, nullptr, nullptr, d, e, -1}};
    int n = 0;
    const int sched = g_schedule.load();
    for_role_groups(is_bwd ? bwd : fwd, is_bwd ? 3 : 1, [&](const RoleDesc* g, int m) {
        if (out && n < max_out) {
            const long long units = static_cast<long long>(B) * H * m;
            SegPlan sp = plan_segments(units, T, sched);
            if (block != la2::ws::kTB) {
                // T_B = 64 / 256: one CTA per (unit, 64 value columns), one segment
                sp = SegPlan();
                sp.seg_tiles = (T + 127) / 128;
                sp.nctas = units * (g[0].dc / la2::blk::kDC);
            }
            la2_plan& o = out[n];
            o.d = g[0].da;
            o.e = g[0].dc;
            o.schedule = sp.balanced ? LA2_SCHEDULE_BALANCED : LA2_SCHEDULE_UNIFORM;
            o.units = units;
            o.segments = sp.balanced ? 0 : sp.nseg;
            o.tiles_per_cta = sp.seg_tiles;
            o.ctas = sp.nctas;
            o.prepass_ctas = sp.npre;
        }
        ++n;
        return LA2_OK;
    });
    return n;
}

la2_status la2_fwd_ex(const void* q, const void* k, const void* v, const float* decay, void* out,
                      const float* init_state, float* final_state, int B, int H, int T, int d,
                      int e, int block, la2_dtype dtype, la2_dtype out_dtype, la2_layout layout,
                      void* workspace, size_t workspace_bytes, la2_stream_t stream) {
    t_last_launches = 0;
    if (layout != LA2_LAYOUT_BHTD && layout != LA2_LAYOUT_BTHD) return LA2_ERR_INVALID_ARG;
    if (out_dtype != LA2_DTYPE_F32 && out_dtype != LA2_DTYPE_BF16) return LA2_ERR_INVALID_ARG;
    bool empty = false;
    la2_status st = common_checks(B, H, T, d, e, block, dtype, &empty);
    if (st != LA2_OK) return st;
    if (out_dtype == LA2_DTYPE_BF16 && dtype != LA2_DTYPE_BF16) return LA2_ERR_UNSUPPORTED;
    if (empty) {
        // no position to process: the final state is the initial one (or 0)
        if (final_state && B > 0 && H > 0) {
            const size_t n = static_cast<size_t>(B) * H * d * e * sizeof(float);
            const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
            const cudaError_t err =
                init_state ? cudaMemcpyAsync(final_state, init_state, n, cudaMemcpyDeviceToDevice, cs)
                           : cudaMemsetAsync(final_state, 0, n, cs);
            if (err != cudaSuccess) return LA2_ERR_CUDA;
        }
        return LA2_OK;
    }
    if (!q || !k || !v || !decay || !out) return LA2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(decay) & 3u) ||
        (reinterpret_cast<uintptr_t>(init_state) & 3u) || (reinterpret_cast<uintptr_t>(final_state) & 3u))
        return LA2_ERR_INVALID_ARG;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return LA2_ERR_INVALID_ARG;
    RoleDesc r = {q, k, v, out, d, e, +1};
    r.init = init_state;
    r.fin = final_state;
    return run_roles(&r, 1, decay, B, H, T, block, dtype, layout == LA2_LAYOUT_BTHD,
                     g_schedule.load(), workspace, workspace_bytes,
                     reinterpret_cast<cudaStream_t>(stream), Hold(), false,
                     out_dtype == LA2_DTYPE_BF16);
}

la2_status la2_fwd_state(const void* q, const void* k, const void* v, const float* decay,
                         void* out, const float* init_state, float* final_state, int B, int H,
                         int T, int d, int e, int block, la2_dtype dtype, void* workspace,
                         size_t workspace_bytes, la2_stream_t stream) {
    return la2_fwd_ex(q, k, v, decay, out, init_state, final_state, B, H, T, d, e, block, dtype,
                      LA2_DTYPE_F32, LA2_LAYOUT_BHTD, workspace, workspace_bytes, stream);
}

la2_status la2_fwd(const void* q, const void* k, const void* v, const float* decay, void* out,
                   int B, int H, int T, int d, int e, int block, la2_dtype dtype,
                   void* workspace, size_t workspace_bytes, la2_stream_t stream) {
    return la2_fwd_state(q, k, v, decay, out, nullptr, nullptr, B, H, T, d, e, block, dtype,
                         workspace, workspace_bytes, stream);
}

la2_status la2_bwd(const void* q, const void* k, const void* v, const float* decay,
                   const void* dout, void* dq, void* dk, void* dv, int B, int H, int T, int d,
                   int e, int block, la2_dtype dtype, void* workspace, size_t workspace_bytes,
                   la2_stream_t stream) {
    return la2_bwd_ex(q, k, v, decay, dout, dq, dk, dv, B, H, T, d, e, block, dtype,
                      LA2_DTYPE_F32, LA2_LAYOUT_BHTD, workspace, workspace_bytes, stream);
}

la2_status la2_bwd_ex(const void* q, const void* k, const void* v, const float* decay,
                      const void* dout, void* dq, void* dk, void* dv, int B, int H, int T, int d,
                      int e, int block, la2_dtype dtype, la2_dtype out_dtype, la2_layout layout,
                      void* workspace, size_t workspace_bytes, la2_stream_t stream) {
    return la2_bwd_state(q, k, v, decay, dout, nullptr, nullptr, dq, dk, dv, nullptr, B, H, T, d,
                         e, block, dtype, out_dtype, layout, workspace, workspace_bytes, stream);
}

la2_status la2_bwd_state(const void* q, const void* k, const void* v, const float* decay,
                         const void* dout, const float* init_state, const float* d_final_state,
                         void* dq, void* dk, void* dv, float* d_init_state, int B, int H, int T,
                         int d, int e, int block, la2_dtype dtype, la2_dtype out_dtype,
                         la2_layout layout, void* workspace, size_t workspace_bytes,
                         la2_stream_t stream) {
    t_last_launches = 0;
    if (layout != LA2_LAYOUT_BHTD && layout != LA2_LAYOUT_BTHD) return LA2_ERR_INVALID_ARG;
    if (out_dtype != LA2_DTYPE_F32 && out_dtype != LA2_DTYPE_BF16) return LA2_ERR_INVALID_ARG;
    bool empty = false;
    la2_status st = common_checks(B, H, T, d, e, block, dtype, &empty);
    if (st != LA2_OK) return st;
    if (out_dtype == LA2_DTYPE_BF16 && dtype != LA2_DTYPE_BF16) return LA2_ERR_UNSUPPORTED;
    const uintptr_t smis = reinterpret_cast<uintptr_t>(init_state) |
                           reinterpret_cast<uintptr_t>(d_final_state) |
                           reinterpret_cast<uintptr_t>(d_init_state);
    if (smis & 3u) return LA2_ERR_INVALID_ARG;
    if (empty) {
        // no position: the final state is the initial one, so its gradient
        // passes through unchanged (or is 0)
        if (d_init_state && B > 0 && H > 0) {
            const size_t n = static_cast<size_t>(B) * H * d * e * sizeof(float);
            const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
            const cudaError_t err =
                d_final_state
                    ? cudaMemcpyAsync(d_init_state, d_final_state, n, cudaMemcpyDeviceToDevice, cs)
                    : cudaMemsetAsync(d_init_state, 0, n, cs);
            if (err != cudaSuccess) return LA2_ERR_CUDA;
        }
        return LA2_OK;
    }
    if (!q || !k || !v || !decay || !dout || !dq || !dk || !dv) return LA2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(decay) & 3u))
        return LA2_ERR_INVALID_ARG;
    // dq = scan(+1; dO, v, k), dk = scan(-1; v, dO, q), dv = scan(-1; k, q, dO).
    // The carried states enter as the scans' initial states: S0^T for dq (a
    // state before position 0), G^T for dk and G for dv (a state entering at
    // position T-1); dS0 is the dv scan's final state (lambda times its state
    // at position 0, which is sum_t lambda^(t+1) q_t dO_t^T + lambda^T G).
    RoleDesc roles[3] = {
        {dout, v, k, dq, e, d, +1},
        {v, dout, q, dk, e, d, -1},
        {k, q, dout, dv, d, e, -1},
    };
    roles[0].init = init_state;
    roles[0].init_t = 1;
    roles[1].init = d_final_state;
    roles[1].init_t = 1;
    roles[2].init = d_final_state;
    roles[2].fin = d_init_state;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return LA2_ERR_INVALID_ARG;
    return run_roles(roles, 3, decay, B, H, T, block, dtype, layout == LA2_LAYOUT_BTHD,
                     g_schedule.load(), workspace, workspace_bytes,
                     reinterpret_cast<cudaStream_t>(stream), Hold(), false,
                     out_dtype == LA2_DTYPE_BF16);
}

la2_status la2_decode(const void* q, const void* k, const void* v, const float* decay,
                      float* state, float* out, int B, int H, int d, int e, la2_dtype dtype,
                      la2_stream_t stream) {
    t_last_launches = 0;
    if (dtype != LA2_DTYPE_F32 && dtype != LA2_DTYPE_BF16) return LA2_ERR_INVALID_ARG;
    if (B < 0 || H < 0 || d <= 0 || e <= 0) return LA2_ERR_INVALID_ARG;
    if (B == 0 || H == 0) return LA2_OK;
    if (d > 4096 || e > 4096) return LA2_ERR_UNSUPPORTED;
    if (static_cast<long long>(B) * H > (1LL << 30)) return LA2_ERR_UNSUPPORTED;
    if (!q || !k || !v || !decay || !state || !out) return LA2_ERR_INVALID_ARG;
    const size_t esz = dtype == LA2_DTYPE_BF16 ? 2 : 4;
    const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                          reinterpret_cast<uintptr_t>(v);
    if ((mis & (esz - 1)) || (reinterpret_cast<uintptr_t>(decay) & 3u) ||
        (reinterpret_cast<uintptr_t>(state) & 3u) || (reinterpret_cast<uintptr_t>(out) & 3u))
        return LA2_ERR_INVALID_ARG;
    const bool vec = (e % 4 == 0) && !(reinterpret_cast<uintptr_t>(state) & 15u);
    const dim3 grid(static_cast<unsigned>(B * H));
    const size_t smem = la2::decode_smem_bytes(d);
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    auto run = [&](auto tin_tag, auto vec_tag) {
        using Tin = decltype(tin_tag);
        constexpr bool kV = decltype(vec_tag)::value;
        const auto* qt = static_cast<const Tin*>(q);
        const auto* kt = static_cast<const Tin*>(k);
        const auto* vt = static_cast<const Tin*>(v);
        la2::la2_decode_kernel<Tin, kV><<<grid, la2::kDecThreads, smem, cs>>>(qt, kt, vt, decay, state, out, H, d,
                                                                          e);
    };
    if (dtype == LA2_DTYPE_BF16) {
        if (vec) run(__nv_bfloat16(), std::true_type());
        else run(__nv_bfloat16(), std::false_type());
    } else {
        if (vec) run(float(), std::true_type());
        else run(float(), std::false_type());
    }
    if (cudaGetLastError() != cudaSuccess) return LA2_ERR_CUDA;
    t_last_launches = 1;
    return LA2_OK;
}

la2_status la2_selftest_timeout(const void* q, const void* k, const void* v, const float* decay,
                                void* out, int T, int d, int e, unsigned limit_us,
                                la2_stream_t stream) {
    t_last_launches = 0;
    if (T < 1 || T > 2 * la2::ws::kTB || limit_us == 0 || limit_us > 1000000u)
        return LA2_ERR_INVALID_ARG;
    bool empty = false;
    const la2_status st = common_checks(1, 1, T, d, e, la2::ws::kTB, LA2_DTYPE_BF16, &empty);
    if (st != LA2_OK) return st;
    if (!q || !k || !v || !decay || !out) return LA2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(decay) & 3u))
        return LA2_ERR_INVALID_ARG;
    int dev = 0;
    int* status = nullptr;
    if (!device_setup(&dev, &status)) return LA2_ERR_CUDA;
    Hold hold;
    hold.flag = never_set_flag();
    hold.ns = static_cast<unsigned long long>(limit_us) * 1000ull;
    if (!hold.flag) return LA2_ERR_CUDA;
    // one sequence of at most two tiles: the uniform plan runs it as one
    // segment, so the scan needs no pre-pass and no workspace (launch_bf16_ws
    // refuses a plan with a pre-pass when it gets none)
    const RoleDesc r = {q, k, v, out, d, e, +1};
    return launch_bf16_ws(&r, 1, decay, 1, 1, T, false, LA2_SCHEDULE_UNIFORM, status, nullptr, hold,
                          reinterpret_cast<cudaStream_t>(stream));
}

size_t la2_dlambda_workspace_bytes(int B, int H, int T, int d, int e, la2_dtype dtype) {
    if (dtype != LA2_DTYPE_F32 && dtype != LA2_DTYPE_BF16) return static_cast<size_t>(-1);
    if (B < 0 || H < 0 || T < 0 || d <= 0 || e <= 0) return static_cast<size_t>(-1);
    if (d > 128 || e > 128 || static_cast<long long>(B) * H > (1LL << 24)) return static_cast<size_t>(-1);
    if (B == 0 || H == 0 || T == 0) return 0;
    return dl_workspace_bytes(static_cast<long long>(B) * H, T, d, e);
}

la2_status la2_dlambda(const void* q, const void* k, const void* v, const float* decay,
                       const void* dout, const float* init_state, const float* d_final_state,
                       float* d_decay, int B, int H, int T, int d, int e, la2_dtype dtype,
                       la2_layout layout, void* workspace, size_t workspace_bytes,
                       la2_stream_t stream) {
    t_last_launches = 0;
    if (dtype != LA2_DTYPE_F32 && dtype != LA2_DTYPE_BF16) return LA2_ERR_INVALID_ARG;
    if (layout != LA2_LAYOUT_BHTD && layout != LA2_LAYOUT_BTHD) return LA2_ERR_INVALID_ARG;
    if (B < 0 || H < 0 || T < 0 || d <= 0 || e <= 0) return LA2_ERR_INVALID_ARG;
    if (d > 128 || e > 128 || static_cast<long long>(B) * H > (1LL << 24)) return LA2_ERR_UNSUPPORTED;
    if (H == 0) return LA2_OK;
    if (!d_decay || (reinterpret_cast<uintptr_t>(d_decay) & 3u)) return LA2_ERR_INVALID_ARG;
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (B == 0 || T == 0) {
        // no position: L does not depend on lambda
        return cudaMemsetAsync(d_decay, 0, static_cast<size_t>(H) * sizeof(float), cs) == cudaSuccess
                   ? LA2_OK
                   : LA2_ERR_CUDA;
    }
    if (!q || !k || !v || !decay || !dout) return LA2_ERR_INVALID_ARG;
    const size_t esz = dtype == LA2_DTYPE_BF16 ? 2 : 4;
    const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                          reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(dout);
    const uintptr_t smis = reinterpret_cast<uintptr_t>(decay) | reinterpret_cast<uintptr_t>(init_state) |
                           reinterpret_cast<uintptr_t>(d_final_state);
    if ((mis & (esz - 1)) || (smis & 3u)) return LA2_ERR_INVALID_ARG;
    const long long seqs = static_cast<long long>(B) * H;
    const size_t need = dl_workspace_bytes(seqs, T, d, e);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u) ? LA2_ERR_INVALID_ARG
                                                                               : LA2_ERR_WORKSPACE;
    int dev = 0;
    int* status = nullptr;
    if (!device_setup(&dev, &status)) return LA2_ERR_CUDA;
    const DlPlan pl = dl_plan(seqs, T);
    la2::DlParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = q;
    p.k = k;
    p.v = v;
    p.g = dout;
    p.decay = decay;
    p.init = init_state;
    p.dfin = d_final_state;
    size_t poff = static_cast<size_t>(seqs) * pl.g * sizeof(double);
    poff = (poff + 255) & ~static_cast<size_t>(255);
    p.partial = static_cast<double*>(workspace);
    p.seg_state = reinterpret_cast<float*>(static_cast<char*>(workspace) + poff);
    p.d_decay = d_decay;
    p.B = B;
    p.H = H;
    p.T = T;
    p.d = d;
    p.e = e;
    p.bthd = layout == LA2_LAYOUT_BTHD ? 1 : 0;
    p.nseg = pl.nseg;
    p.seg_rows = pl.seg_rows;
    // 16-byte vector staging when every row starts on a 16-byte boundary
    const int vel = static_cast<int>(16 / esz);
    p.vec = (d % vel == 0 && e % vel == 0 && !(mis & 15u)) ? 1 : 0;
    const bool bf = dtype == LA2_DTYPE_BF16;
    int launches = 0;
    if (pl.nseg > 1) {
        const unsigned grid = static_cast<unsigned>(seqs * (pl.nseg - 1));
        if (bf)
            la2::la2_dlam_prepass<__nv_bfloat16><<<grid, la2::kDlThreads, la2::dl_prepass_smem_bytes(), cs>>>(p);
        else
            la2::la2_dlam_prepass<float><<<grid, la2::kDlThreads, la2::dl_prepass_smem_bytes(), cs>>>(p);
        ++launches;
    }
    const unsigned grid = static_cast<unsigned>(seqs * pl.nseg);
    if (bf)
        la2::la2_dlam_scan<__nv_bfloat16><<<grid, la2::kDlThreads, la2::dl_scan_smem_bytes(), cs>>>(p);
    else
        la2::la2_dlam_scan<float><<<grid, la2::kDlThreads, la2::dl_scan_smem_bytes(), cs>>>(p);
    la2::la2_dlam_reduce<<<static_cast<unsigned>((H + 255) / 256), 256, 0, cs>>>(p);
    launches += 2;
    if (cudaGetLastError() != cudaSuccess) return LA2_ERR_CUDA;
    t_last_launches = launches;
    return LA2_OK;
}


size_t la2_norm_workspace_bytes(int B, int H, int T, int d, int e, int block, la2_dtype dtype,
                                int is_bwd) {
    bool empty = false;
    if (common_checks(B, H, T, d, e, block, dtype, &empty) != LA2_OK || d > 128)
        return static_cast<size_t>(-1);
    if (empty) return 0;
    const long long seqs = static_cast<long long>(B) * H;
    size_t n = align256(la2_workspace_bytes(B, H, T, d, e, block, dtype, is_bwd));
    if (is_bwd) n += 2 * align256(static_cast<size_t>(seqs) * T * sizeof(float));
    return n + nz_chunk_bytes(seqs, T, d);
}

la2_status la2_fwd_norm(const void* q, const void* k, const void* v, const float* decay, float* y,
                        float* den, int B, int H, int T, int d, int e, int block, la2_dtype dtype,
                        la2_layout layout, void* workspace, size_t workspace_bytes,
                        la2_stream_t stream) {
    t_last_launches = 0;
    bool empty = false;
    la2_status st = norm_checks(q, k, v, decay, B, H, T, d, e, block, dtype, layout, &empty);
    if (st != LA2_OK || empty) return st;
    if (!y || (reinterpret_cast<uintptr_t>(den) & 3u)) return LA2_ERR_INVALID_ARG;
    const size_t need = la2_norm_workspace_bytes(B, H, T, d, e, block, dtype, 0);
    if (need > 0 && (!workspace || workspace_bytes < need)) return LA2_ERR_WORKSPACE;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return LA2_ERR_INVALID_ARG;
    const size_t fws = align256(la2_workspace_bytes(B, H, T, d, e, block, dtype, 0));
    // the numerator (the normalised form's instantiation: hi + lo operands at every (d, e))
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(y) ||
        (reinterpret_cast<uintptr_t>(decay) & 3u))
        return LA2_ERR_INVALID_ARG;
    const RoleDesc num = {q, k, v, y, d, e, +1};
    st = run_roles(&num, 1, decay, B, H, T, block, dtype, layout == LA2_LAYOUT_BTHD,
                   g_schedule.load(), fws ? workspace : nullptr, fws,
                   reinterpret_cast<cudaStream_t>(stream), Hold(), true);
    if (st != LA2_OK) return st;
    int launches = t_last_launches;
    // the denominator, dividing y in place
    char* base = static_cast<char*>(workspace);
    la2::NzParams p = nz_params(B, H, T, d, e, layout == LA2_LAYOUT_BTHD, decay,
                                base ? reinterpret_cast<float*>(base + fws) : nullptr);
    p.a = k;
    p.q = q;
    p.y = y;
    p.den = den;
    p.mode = la2::kNzDen;
    p.dir = +1;
    if (p.nchunk > 1 && !p.chunk) return LA2_ERR_WORKSPACE;
    const long long seqs = static_cast<long long>(B) * H;
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == LA2_DTYPE_BF16) nz_launch<__nv_bfloat16>(p, seqs, cs, &launches);
    else nz_launch<float>(p, seqs, cs, &launches);
    if (cudaGetLastError() != cudaSuccess) return LA2_ERR_CUDA;
    t_last_launches = launches;
    return LA2_OK;
}

la2_status la2_bwd_norm(const void* q, const void* k, const void* v, const float* decay,
                        const float* y, const float* den, const void* dy, void* dq, void* dk,
                        void* dv, int B, int H, int T, int d, int e, int block, la2_dtype dtype,
                        la2_layout layout, void* workspace, size_t workspace_bytes,
                        la2_stream_t stream) {
    t_last_launches = 0;
    bool empty = false;
    la2_status st = norm_checks(q, k, v, decay, B, H, T, d, e, block, dtype, layout, &empty);
    if (st != LA2_OK || empty) return st;
    if (!y || !den || !dy || !dq || !dk || !dv) return LA2_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dy) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(decay) & 3u) ||
        (reinterpret_cast<uintptr_t>(y) & 3u) || (reinterpret_cast<uintptr_t>(den) & 3u))
        return LA2_ERR_INVALID_ARG;
    const size_t need = la2_norm_workspace_bytes(B, H, T, d, e, block, dtype, 1);
    if (!workspace || workspace_bytes < need) return LA2_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return LA2_ERR_INVALID_ARG;
    int dev = 0;
    int* status = nullptr;
    if (!device_setup(&dev, &status)) return LA2_ERR_CUDA;
    const long long seqs = static_cast<long long>(B) * H;
    const size_t bws = align256(la2_workspace_bytes(B, H, T, d, e, block, dtype, 1));
    const size_t rows = align256(static_cast<size_t>(seqs) * T * sizeof(float));
    char* base = static_cast<char*>(workspace);
    float* dden = reinterpret_cast<float*>(base + bws);
    float* inv = reinterpret_cast<float*>(base + bws + rows);
    float* chunk = reinterpret_cast<float*>(base + bws + 2 * rows);
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const bool bthd = layout == LA2_LAYOUT_BTHD;
    int launches = 0;
    // dden_t = -(dy_t . y_t) / den_t, inv_t = 1 / den_t
    {
        const long long nrows = seqs * T;
        const unsigned grid = static_cast<unsigned>(cdiv(nrows * 32, 256));
        if (dtype == LA2_DTYPE_BF16)
            la2::la2_nz_prep<__nv_bfloat16><<<grid, 256, 0, cs>>>(static_cast<const __nv_bfloat16*>(dy), y,
                                                                   den, dden, inv, nrows, H, T, e, bthd);
        else
            la2::la2_nz_prep<float><<<grid, 256, 0, cs>>>(static_cast<const float*>(dy), y, den, dden, inv,
                                                          nrows, H, T, e, bthd);
        ++launches;
        if (cudaGetLastError() != cudaSuccess) return LA2_ERR_CUDA;
    }
    // the numerator's backward with dnum_t = dy_t / den_t: the dq scan with
    // dout = dy (its rows are divided by den_t afterwards), the dk and dv scans
    // with the factor 1 / den_t on their summed position
    RoleDesc roles[3] = {
        {dy, v, k, dq, e, d, +1},
        {v, dy, q, dk, e, d, -1},
        {k, q, dy, dv, d, e, -1},
    };
    roles[1].colf = inv;
    roles[2].colf = inv;
    st = run_roles(roles, 3, decay, B, H, T, block, dtype, bthd, g_schedule.load(),
                   bws ? workspace : nullptr, bws, cs, Hold(), true);
    if (st != LA2_OK) return st;
    launches += t_last_launches;
    // dq_t = dq_t / den_t + dden_t z_t, then dk_s += sum_{t>=s} lambda^(t-s) dden_t q_t
    la2::NzParams p = nz_params(B, H, T, d, e, bthd, decay, chunk);
    p.w = dden;
    p.rs = inv;
    p.a = k;
    p.out = static_cast<float*>(dq);
    p.mode = la2::kNzDq;
    p.dir = +1;
    if (dtype == LA2_DTYPE_BF16) nz_launch<__nv_bfloat16>(p, seqs, cs, &launches);
    else nz_launch<float>(p, seqs, cs, &launches);
    p.a = q;
    p.out = static_cast<float*>(dk);
    p.mode = la2::kNzDk;
    p.dir = -1;
    if (dtype == LA2_DTYPE_BF16) nz_launch<__nv_bfloat16>(p, seqs, cs, &launches);
    else nz_launch<float>(p, seqs, cs, &launches);
    if (cudaGetLastError() != cudaSuccess) return LA2_ERR_CUDA;
    t_last_launches = launches;
    return LA2_OK;
}

const char* la2_status_str(la2_status s) {
    switch (s) {
        case LA2_OK: return "LA2_OK";
        case LA2_ERR_INVALID_ARG: return "LA2_ERR_INVALID_ARG";
        case LA2_ERR_UNSUPPORTED: return "LA2_ERR_UNSUPPORTED";
        case LA2_ERR_WORKSPACE: return "LA2_ERR_WORKSPACE";
        case LA2_ERR_CUDA: return "LA2_ERR_CUDA";
        case LA2_ERR_TIMEOUT: return "LA2_ERR_TIMEOUT";
    }
    return "LA2_UNKNOWN_STATUS";
}

la2_status la2_device_status(int* code, int reset) {
    if (!code) return LA2_ERR_INVALID_ARG;
    int dev = 0;
    int* status = nullptr;
    if (!device_setup(&dev, &status)) return LA2_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return LA2_ERR_CUDA;
    if (cudaMemcpy(code, status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return LA2_ERR_CUDA;
    if (reset) {
        const int zero = 0;
        if (cudaMemcpy(status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
            return LA2_ERR_CUDA;
    }
    return LA2_OK;
}

int la2_last_launch_count(void) { return t_last_launches; }

#ifdef LA2_TRACE
// Debug builds only: copies (and clears) the timeline trace of la2_scan_ws.
int la2_trace_read(void* host, size_t bytes) {
    constexpr size_t kTraceBytes = sizeof(unsigned long long) * 2 * la2::ws::kTraceEv *
                                   la2::ws::kTraceSteps;
    static unsigned long long zero[kTraceBytes / 8];
    if (bytes > kTraceBytes) bytes = kTraceBytes;
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    if (cudaMemcpyFromSymbol(host, la2::ws::g_la2_trace, bytes) != cudaSuccess) return -1;
    if (cudaMemcpyToSymbol(la2::ws::g_la2_trace, zero, kTraceBytes) != cudaSuccess) return -1;
    return static_cast<int>(bytes);
}
#endif

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free forward: the segment states live in a fixed array that is
// part of the library image on every GPU that loads it, instead of in a
// caller-provided workspace.
namespace {

// Large enough for any forward call: the segment states of one call never
// exceed 147 units of d x e fp32 (148 CTAs at most, and the last segment of
// every sequence needs none), i.e. 147 * 128 * 128 * 4 bytes at d = e = 128.
constexpr size_t kStaticScratchBytes = static_cast<size_t>(148) * 128 * 128 * 4;

static __device__ __align__(256) unsigned char g_la2_static_scratch[kStaticScratchBytes];

struct ScratchState {
    std::once_flag once;
    void* ptr = nullptr;
    bool ok = false;
};
ScratchState g_scratch[kMaxDevices];

// Device address of the scratch array on the current device.  The host-side
// symbol is only a stand-in; the address must come from cudaGetSymbolAddress,
// once per device, with that device current.
void* static_scratch_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    ScratchState& s = g_scratch[dev];
    std::call_once(s.once, [&s] {
        void* ptr = nullptr;
        s.ok = cudaGetSymbolAddress(&ptr, g_la2_static_scratch) == cudaSuccess;
        s.ptr = ptr;
    });
    return s.ok ? s.ptr : nullptr;
}

}  // namespace

extern "C" la2_status la2_fwd_noalloc(const void* q, const void* k, const void* v,
                                      const float* decay, void* out, int B, int H, int T, int d,
                                      int e, int block, la2_dtype dtype, la2_stream_t stream) {
    t_last_launches = 0;
    bool empty = false;
    la2_status st = common_checks(B, H, T, d, e, block, dtype, &empty);
    if (st != LA2_OK || empty) return st;
    const size_t need = la2_workspace_bytes(B, H, T, d, e, block, dtype, 0);
    if (need > kStaticScratchBytes) return LA2_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (need > 0) {
        scratch = static_scratch_ptr();
        if (!scratch) return LA2_ERR_CUDA;
    }
    return la2_fwd(q, k, v, decay, out, B, H, T, d, e, block, dtype, scratch,
                   need > 0 ? kStaticScratchBytes : 0, stream);
}
