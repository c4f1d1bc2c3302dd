// scan_ws_sm100.cuh -- warp-specialised bf16-input tcgen05 kernel of the
// Lightning Attention-2 hot path: one CTA per SM, running one segment of one
// (sequence, role) unit (or, in the balanced schedule, the pieces of several
// units one after the other), the whole value width (DC = 64 or 128) in one
// CTA, tiles of T_B = 128 rows.
//
// It computes the same decayed scan as the forward and backward roles of the
// library (see la2_api.cu):
//
//   dir = +1:  x_t = sum_{s<=t} lambda^(t-s) (a_t . b_s) c_s
//   dir = -1:  x_t = sum_{s>=t} lambda^(s-t) (a_t . b_s) c_s
//
// following the tiled derivation of the "Lightning Attention" page
// (lizeman.github.io llm-arch-kb, section 2, steps 1-4) with the decay folded
// in.  Per tile i (local row r, column c):
//
//   S   = A_i B_i^T                                 (tcgen05, TMEM)
//   P   = S * lambda^|r-c| on the causal side, else 0 (registers -> TMEM)
//   X   = diag(w_x) A_i W + P C_i                   (tcgen05, TMEM, fp32)
//   dW  = (diag(w_s) B_i)^T C_i                     (tcgen05, TMEM)
//   W  <- lambda^T_B W + dW                         (fp32 arithmetic)
//
// with w_x = lambda^(r+1), w_s = lambda^(T_B-1-r) for dir = +1 and
// w_x = lambda^(T_B-r), w_s = lambda^r for dir = -1.  Operand precision: at
// DA = DC = 64, P and w_s B enter their MMAs as tf32 (P stays fp32 in TMEM;
// the mask warps write fp32 copies of C and w_s B, transposed so that they are
// K-major); otherwise P and w_s B are split into bf16 hi + lo pairs.  The
// state W is always kept as its bf16 hi + lo pair in shared memory (the X
// MMA's operand), and in fp32 registers as well at DC = 64.
//
// Roles (20 warps):
//   warp 0      TMA producer and MMA issuer S, one polling loop: A, B and C
//               each in a ring of buffers (whichever ring has a free buffer is
//               refilled first), S = A B^T into S buffer s % 2
//   warp 1      MMA issuer PC: X += P C, P read from S buffer s % 2 as the
//               TMEM A operand
//   warp 2      MMA issuer XW: A W, into X_inter (DC = 64) or into X (DC = 128)
//   warp 3      MMA issuer dW
//   warps 4-11  mask group (two warps per TMEM lane quadrant): the operand
//               copies or hi/lo splits of C and w_s B, then P from S
//   warps 12-19 epilogue group (two warps per lane quadrant, one per half of
//               the columns): the W update, and the output: X (+ w_x X_inter
//               at DC = 64) read with the 16x256b TMEM shape, so that float2
//               stores of a warp fill whole 32-byte sectors
// The tensor core takes one N = 64 MMA about every 45 cycles and one N = 128
// MMA every 64, but a single issuing thread is slower than that once it also
// computes descriptors and waits, so the MMAs of a tile are spread over four
// issuing threads; at d = 64 those warps run their loops warp-converged (lane
// 0 issues through predicated instructions).
// How many buffers each operand gets depends on (DA, DC) (RingCfg): shared
// memory holds two of most rings, and at DA = DC = 128 one A, C and W buffer
// and two B buffers.  With DC = 64, X += P C, X_inter (two buffers) and dW
// are separate TMEM accumulators; otherwise A W is scaled in place by w_x
// before P C adds to it (one X buffer), and the fp32 state itself sits in
// TMEM, dW accumulating onto it.
//
// Every hand-off is an mbarrier: each buffer has a "full" barrier its
// producer completes and an "empty" barrier its consumers complete, so a
// waiter is never more than one phase behind.  Every wait is bounded (2 s) and
// a shared abort flag stops all roles once one of them gives up, after which
// the kernel waits (bounded) for its own MMAs, frees TMEM and returns.
#pragma once
#include "ptx_sm100.cuh"

namespace la2 {
namespace ws {

constexpr int kTB = 128;
constexpr int kThreads = 640;
constexpr uint32_t kTmemCols = 512;

struct Role {
    CUtensorMap ta, tb, tc;  // a, b: 4-D maps of [B, H, T, DA] (or [B, T, H, DA]); c likewise
                             // with DC; bf16, box 64 columns x 128 positions
    void* x;                 // [B*H, T, DC] fp32, or bf16 in the kXb16 instantiation
    const float* init;       // [B*H, DA, DC] fp32 state the scan starts from, or null (0);
                             // with init_t, [B*H, DC, DA] read transposed
    float* fin;              // [B*H, DA, DC] fp32 state the scan ends with, or null
    int dir;                 // +1 or -1
    int init_t;              // 1: init is stored transposed
    const float* colf;       // [B*H, T] fp32 factor f_s on the summed position s, or null (1):
                             // x_t = sum_s lambda^|t-s| (a_t . b_s) f_s c_s, applied in fp32 to
                             // the columns of P and to the state-update weights of row s
    // dir = +1: init is the state before position 0 (row t of the output gets
    // lambda^(t+1) a_t^T init) and fin the state after position T-1.
    // dir = -1: init is a state entering at position T-1 (row t gets
    // lambda^(T-1-t) a_t^T init), and fin is lambda times the state at
    // position 0, i.e. the state the scan would carry past the first position.
};

struct Params {
    Role role[3];
    const float* decay;  // [H]
    int* status;         // device status word
    float* seg_state;    // [slots][DA][DC] fp32: local end state of each segment but the
                         // last of its unit (written by the state pass), see seg_slot_index
    int H, T, nroles;
    int bthd;            // 0: tensors [B, H, T, D]; 1: [B, T, H, D] (rows of a sequence H*D apart)
    int nunits;          // (sequence, role) units, unit u = (sequence u / nroles, role u % nroles)
    int seg_tiles;       // L: segment length in tiles
    int balanced;        // 0: every unit is cut into nseg segments [j L, (j+1) L), one CTA
                         //    each (CTA c: unit c / nseg, segment c % nseg);
                         // 1: the units' steps laid end to end, CTA c takes global steps
                         //    [c L, (c+1) L), i.e. the ends of some units and the starts
                         //    of others, one after the other
    int nseg;            // balanced = 0: segments per unit (1 = no split)
    const int* hold;     // null, except in the failure-path self-test: a device flag that
                         // nothing sets, which the producer waits on (bounded by hold_ns)
                         // before its first load, so that the wait runs out
    unsigned long long hold_ns;
};

// Status code a kernel records when a bounded wait runs out: LA2_ERR_TIMEOUT
// (5) in the low byte, the site of the wait above it.
constexpr int kTimeoutCode = 5;
constexpr int kSiteHold = 90;  // the self-test's wait on p.hold

// Segments of unit u (nb tiles, in scan order).  Boundary j >= 1 sits at step
// j L - ph(u), where ph(u) = (u nb) mod L in the balanced plan (the boundaries
// are the CTA boundaries of the global step axis) and 0 otherwise.
// (`balanced` is p.balanced, passed separately so that a kernel that knows it
// at compile time drops the other branch.)
__device__ __forceinline__ int seg_phase(const Params& p, bool balanced, int u, int nb) {
    return balanced ? static_cast<int>((static_cast<long long>(u) * nb) % p.seg_tiles) : 0;
}
__device__ __forceinline__ int seg_begin(const Params& p, bool balanced, int u, int j, int nb) {
    return j == 0 ? 0 : min(nb, j * p.seg_tiles - seg_phase(p, balanced, u, nb));
}
// Slot in seg_state of segment j (not the unit's last): balanced, the index of
// the CTA boundary that ends it, minus one; otherwise u (nseg - 1) + j.
__device__ __forceinline__ long long seg_slot_index(const Params& p, bool balanced, int u, int j, int nb) {
    return balanced ? static_cast<long long>(u) * nb / p.seg_tiles + j
                    : static_cast<long long>(u) * (p.nseg - 1) + j;
}

// Buffer counts and mbarrier indices of the scan kernel for (DA, DC).
//
// Two operand modes.  At DA = DC = 64 (kTf32) shared memory has room for fp32
// copies of C and of w_s B, so P (fp32 in TMEM) and w_s B enter their MMAs as
// tf32: no hi/lo split, and w_s B is written to its own buffer, so it need
// not wait for S.  Otherwise P and w_s B are bf16 hi + lo pairs (hi of w_s B
// in place of B).  The state W is a bf16 hi + lo pair in both modes.
//
// kNorm is the instantiation the normalised form uses.  It forces the bf16
// hi + lo mode at DA = DC = 64 as well (about 1e-5 instead of 2e-3 of rms):
// the normalised form divides by q . z and its backward subtracts nearly equal
// parts, which would magnify tf32's error.  It alone compiles the per-position
// factor (Role::colf), so the other instantiations carry none of its code.
template <int DA, int DC, bool kNorm = false>
struct RingCfg {
    static constexpr bool kTf32 = DA == 64 && DC == 64 && !kNorm;
    static constexpr bool kBig = DA == 128 && DC == 128;
    static constexpr int NA = kBig ? 1 : 2;                  // A tiles
    static constexpr int NB = 2;                             // B tiles
    static constexpr int NC = kBig ? 1 : 2;                  // C tiles (bf16, as loaded)
    static constexpr int NBLO = kTf32 ? 0 : (DA == 64 ? 2 : 1);  // lo(w_s B) (bf16 mode)
    static constexpr int NCF = kTf32 ? 2 : 0;                // fp32 C (tf32 mode)
    static constexpr int NWB = kTf32 ? 1 : 0;                // fp32 w_s B (tf32 mode)
    static constexpr int NW = DA == 64 ? 2 : 1;              // W as its hi/lo pair
    // DC = 64 (kOwnD): X += P C (one TMEM buffer), X_inter = A W (two) and
    // dW (one) are separate accumulators, and the epilogue forms
    // w_x X_inter + X; X += P C then never waits for the state, and X_inter
    // of tile s never waits for the output of tile s-1.  DC = 128 (kWT): X
    // (one buffer) holds A W, scaled by w_x in TMEM, then P C; the state W
    // itself lives in TMEM in fp32 (128 columns): the epilogue writes
    // lambda^T_B W back after reading W for its hi/lo pair, and dW of the
    // next tile accumulates onto it, so W <- lambda^T_B W + dW costs no
    // shared-memory read of the state and dW never waits for the output.
    static constexpr bool kOwnD = DC == 64;
    static constexpr bool kWT = DC == 128;
    static constexpr int ND = 1;                             // dW accumulators (own-D)
    static constexpr int NX = 1;                             // X accumulators in TMEM
    static constexpr int NXW = kOwnD ? 2 : NX;               // XW_DONE barriers
    static constexpr int NXS = kOwnD ? 0 : NX;               // XS barriers (scaled in TMEM)
    static constexpr int NXI = kOwnD ? 2 : 0;                // X_inter buffers (EMPTY_XI: read out)
    static constexpr int NBS = kTf32 ? 0 : NB;
    // "full": the producer has filled the buffer; "empty": its consumers are done
    static constexpr int FULL_A = 0, EMPTY_A = FULL_A + NA;
    static constexpr int FULL_B = EMPTY_A + NA, EMPTY_B = FULL_B + NB, BS = EMPTY_B + NB;
    static constexpr int FULL_C = BS + NBS, EMPTY_C = FULL_C + NC;
    static constexpr int EMPTY_BLO = EMPTY_C + NC;
    static constexpr int CF_READY = EMPTY_BLO + NBLO, EMPTY_CF = CF_READY + NCF;
    static constexpr int WB_READY = EMPTY_CF + NCF, EMPTY_WB = WB_READY + NWB;
    static constexpr int S_DONE = EMPTY_WB + NWB, EMPTY_S = S_DONE + 2, P_READY = EMPTY_S + 2;
    static constexpr int XW_DONE = P_READY + 2, XS = XW_DONE + NXW, PC_DONE = XS + NXS;
    static constexpr int EMPTY_X = PC_DONE + NX, EMPTY_XI = EMPTY_X + NX;
    static constexpr int D_DONE = EMPTY_XI + NXI, EMPTY_D = D_DONE + ND;
    static constexpr int W_READY = EMPTY_D + ND, EMPTY_W = W_READY + NW;
    static constexpr int FIN = EMPTY_W + NW, NBARS = FIN + 1;

    // arrivals that complete one phase of barrier b
    static __device__ __forceinline__ uint32_t count(int b) {
        if (b >= EMPTY_A && b < EMPTY_A + NA) return 2;   // S and XW commits
        if (b >= EMPTY_B && b < EMPTY_B + NB)             // tf32: S commit + mask reads;
            return kTf32 ? 257 : 1;                        // bf16: dW commit
        if (b >= EMPTY_C && b < EMPTY_C + NC)             // tf32: mask (to fp32);
            return kTf32 ? 256 : 2;                        // bf16: PC and dW commits
        if (b >= EMPTY_CF && b < EMPTY_CF + NCF) return 2; // PC and dW commits
        if (b >= CF_READY && b < CF_READY + NCF) return 256;
        if (b >= WB_READY && b < WB_READY + NWB) return 256;
        if (b >= BS && b < BS + NBS) return 256;          // mask group
        if (b >= P_READY && b < P_READY + 2) return 256;  // mask group
        if (b >= XS && b < XS + NXS) return 256;          // epilogue group
        if (b >= EMPTY_X && b < EMPTY_X + NX) return 256; // epilogue group
        if (b >= EMPTY_XI && b < EMPTY_XI + NXI) return 256;  // epilogue group
        if (b >= EMPTY_D && b < EMPTY_D + ND) return 256; // epilogue group
        if (b >= W_READY && b < W_READY + NW) return 256; // epilogue group
        if (b == FIN) return 4;                           // the four issuers
        return 1;                                         // TMA or one commit
    }
};

template <int DA, int DC, bool kNorm = false>
struct Smem {
    using Q = RingCfg<DA, DC, kNorm>;
    static constexpr uint32_t kAsz = kTB * DA * 2;            // one A (or B) tile
    static constexpr uint32_t kBsz = kAsz;
    static constexpr uint32_t kCsz = kTB * DC * 2;            // one C tile
    static constexpr uint32_t kWsz = DA * DC * 2;             // hi(W) or lo(W)
    static constexpr uint32_t kA = 0;                         // A ring
    static constexpr uint32_t kB = kA + Q::NA * kAsz;         // B ring, each then hi(w_s B)
    static constexpr uint32_t kBlo = kB + Q::NB * kBsz;       // lo(w_s B) ring
    static constexpr uint32_t kC = kBlo + Q::NBLO * kBsz;     // C ring
    // tf32 mode: fp32 C^T and (w_s B)^T, K-major (time contiguous in 128-byte
    // rows, one row per feature), in four 32-step groups of DC (DA) rows each
    static constexpr uint32_t kCFsz = kTB * DC * 4;           // fp32 C^T
    static constexpr uint32_t kWBsz = kTB * DA * 4;           // fp32 (w_s B)^T
    static constexpr uint32_t kCF = kC + Q::NC * kCsz;        // fp32 C ring (tf32 mode)
    static constexpr uint32_t kWB = kCF + Q::NCF * kCFsz;     // fp32 w_s B ring (tf32 mode)
    static constexpr uint32_t kW = kWB + Q::NWB * kWBsz;      // W buffer i: hi, then lo
    static constexpr uint32_t kPow = kW + Q::NW * 2 * kWsz;   // lambda^n, n = 0..T_B
    static constexpr uint32_t kMuRev = kPow + 528;            // lambda^(15-n), n = 0..15
    static constexpr uint32_t kZ = kMuRev + 64;               // diagonal-block weights, 4 shifted copies
    static constexpr uint32_t kZstride = 72 * 4;              // bytes per copy (72 = 8 mod 32 floats)
    static constexpr uint32_t kBar = kZ + 4 * kZstride;
    static constexpr uint32_t kTmemSlot = kBar + 2 * Q::NBARS * 8;  // two barrier sets
    static constexpr uint32_t kAbort = kTmemSlot + 4;
    static constexpr uint32_t kBytes = kAbort + 12;
    static_assert(kBytes <= 232448, "shared memory over the 227 KB per-CTA limit");
    // one CTA per SM: it allocates all 512 TMEM columns
    static_assert(kBytes > 116 * 1024, "two CTAs would fit on an SM");
};

// Byte offset of the 16-byte chunk q (0..7) of row r inside a 128-byte
// swizzled region (rows of 128 bytes, 8-row groups of 1024 bytes).
__device__ __forceinline__ uint32_t sw128(int r, int q) {
    return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((q ^ (r & 7)) << 4));
}

#ifdef LA2_TRACE
// Timeline trace, compiled only with -DLA2_TRACE (never in the library build):
// clock64() at fixed points of each role, per step, for two CTAs (the first
// and the middle one of the grid), read back with la2_trace_read().
constexpr int kTraceEv = 32, kTraceSteps = 64;
__device__ unsigned long long g_la2_trace[2][kTraceEv][kTraceSteps];
#define LA2_TR(ev, s)                                                                   \
    do {                                                                                \
        const int c_ = blockIdx.x == 0 ? 0 : (blockIdx.x == gridDim.x / 2 ? 1 : -1);   \
        if (c_ >= 0 && (s) >= 0 && (s) < kTraceSteps) g_la2_trace[c_][ev][s] = clock64(); \
    } while (0)
#else
#define LA2_TR(ev, s) ((void)0)
#endif

// TMA load of the 64-column x 128-position box at column x, position t of
// sequence bh, from a 4-D map laid out (D, T, H, B) or, with bthd, (D, H, T, B).
__device__ __forceinline__ void load_box(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x,
                                         int t, int bh, int H, int bthd) {
    const int b = bh / H, h = bh - b * H;
    if (bthd) tma_load_4d(dst, map, bar, x, h, t, b);
    else tma_load_4d(dst, map, bar, x, t, h, b);
}
__device__ __forceinline__ void prefetch_box(const CUtensorMap* map, int x, int t, int bh, int H, int bthd) {
    const int b = bh / H, h = bh - b * H;
    if (bthd) tma_prefetch_4d(map, x, h, t, b);
    else tma_prefetch_4d(map, x, t, h, b);
}

// Bounded wait that also gives up as soon as another role has aborted.  The
// loop is kept out of line (one copy for every call site) to keep each role's
// code small; the first probe is inline.
__device__ __noinline__ bool wait_bar_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           int* status, int where) {
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_try_wait_hint(bar, parity, 64)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > 2000000000ull) {
            *abort_flag = 1;
            atomicCAS(status, 0, 5 | (where << 8));
            return false;
        }
    }
}

// kOutline: the retry loop out of line (measured faster where instruction
// fetch limits the kernel, d = 64) or inline (d = 128).
template <bool kOutline = false>
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         int* status, int where) {
    if (mbar_try_wait_hint(bar, parity, 64)) return true;
    if constexpr (kOutline) return wait_bar_slow(bar, parity, abort_flag, status, where);
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_try_wait_hint(bar, parity, 64)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > 2000000000ull) {
            *abort_flag = 1;
            atomicCAS(status, 0, 5 | (where << 8));
            return false;
        }
    }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}

// Phase parity of the barrier of a ring of n buffers that step s waits for:
// full_par, the fill for step s; empty_par (s >= n), the release by step s - n.
__device__ __forceinline__ uint32_t full_par(int s, int n) { return static_cast<uint32_t>((s / n) & 1); }
__device__ __forceinline__ uint32_t empty_par(int s, int n) {
    return static_cast<uint32_t>(((s / n) + 1) & 1);
}

// The scan itself.  A segment j of a (sequence, role) unit starts from the
// state the segments before it leave behind, W_in(j) = f_{j-1} W_in(j-1) +
// S_{j-1} with f_i = lambda^(T_B n_i) (n_i tiles in segment i) and W_in(0) the
// given initial state or 0; the S_i are read from seg_state (written by
// la2_state_ws).
// kMulti: the balanced plan's CTAs, which may run several segments (a
// separate instantiation, so that the one-segment kernel carries no loop
// state in its registers).
// kXb16: the outputs are bf16, each fp32 result rounded to nearest even once
// in the output epilogue (a separate instantiation: a run-time choice between
// the two store loops measured 6% slower at d = 64, where instruction fetch
// limits the kernel).
template <int DA, int DC, bool kMulti, bool kNorm = false, bool kXb16 = false>
__global__ void __launch_bounds__(kThreads, 1)
la2_scan_ws(const __grid_constant__ Params p)
{
    static_assert((DA == 64 || DA == 128) && (DC == 64 || DC == 128), "DA, DC in {64, 128}");
    using L = Smem<DA, DC, kNorm>;
    using Q = RingCfg<DA, DC, kNorm>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    if (base & 1023u) {  // 128-byte swizzled tiles need a 1024-byte aligned base
        if (threadIdx.x == 0) atomicCAS(p.status, 0, 4);  // LA2_ERR_CUDA
        return;
    }
    const uint32_t sA = base + L::kA, sB = base + L::kB, sBlo = base + L::kBlo;
    const uint32_t sC = base + L::kC, sW = base + L::kW;
    const uint32_t sCF = base + L::kCF, sWB = base + L::kWB;
    float* pw = reinterpret_cast<float*>(smem_raw + L::kPow);
    float* murev = reinterpret_cast<float*>(smem_raw + L::kMuRev);
    // Two sets of barriers: segment i of a CTA uses set i % 2, so that a set
    // is initialised again only after a whole segment has run since its last
    // use (no arrival of a finished segment can still be on its way then).
    uint32_t bar_set = base + L::kBar;
    auto bar = [&](int b) { return bar_set + 8u * b; };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem_raw + L::kAbort);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = p.T;
    const int nb = (T + kTB - 1) / kTB;

    if (tid == 0) LA2_TR(0, 0);
    // ---- set-up: TMEM and barriers here; the decay tables and W buffer 0 are
    // made below by the mask and epilogue warps (the only ones that read them),
    // while the producer's first loads are already in flight
    if (warp == 0) {
        tmem_alloc(base + L::kTmemSlot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int b = 0; b < (kMulti ? 2 : 1) * Q::NBARS; ++b) mbar_init(bar(b), Q::count(b % Q::NBARS));
        *abort_flag = 0;
        fence_mbar_init();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (tid == 0) LA2_TR(1, 0);
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem_raw + L::kTmemSlot);

    // ---- the CTA's segments, one after the other: one in the uniform plan;
    // in the balanced plan the pieces of the units its global steps cover
    for (int item = 0; item < (kMulti ? 0x7fffffff : 1); ++item) {
    int unit, sj, s0, ns;  // (sequence, role), segment, its steps [s0, s0 + ns)
    if (!kMulti) {
        unit = blockIdx.x / p.nseg;
        sj = blockIdx.x % p.nseg;
        s0 = seg_begin(p, kMulti, unit, sj, nb);
        ns = max(0, seg_begin(p, kMulti, unit, sj + 1, nb) - s0);
    } else {
        // global steps [c0, c1) of this CTA; item i is the piece of unit
        // c0 / nb + i they cover
        const long long c0 = static_cast<long long>(blockIdx.x) * p.seg_tiles;
        const long long c1 = min(c0 + p.seg_tiles, static_cast<long long>(p.nunits) * nb);
        unit = static_cast<int>(c0 / nb) + item;
        const long long ub = static_cast<long long>(unit) * nb;
        if (ub >= c1) break;
        s0 = static_cast<int>(max(c0 - ub, 0LL));
        ns = static_cast<int>(min(static_cast<long long>(nb), c1 - ub)) - s0;
        sj = (s0 + seg_phase(p, kMulti, unit, nb)) / p.seg_tiles;
    }
    bar_set = base + L::kBar + static_cast<uint32_t>(item & 1) * (Q::NBARS * 8);
    if (item > 1) {
        // set item % 2 was last used two segments ago: fresh barriers
        if (tid == 0) {
            for (int b = 0; b < Q::NBARS; ++b) {
                mbar_inval(bar(b));
                mbar_init(bar(b), Q::count(b));
            }
            fence_mbar_init();
        }
        __syncthreads();
    }
    const int role_id = unit % p.nroles;
    const int bh = unit / p.nroles;
    const Role& R = p.role[role_id];
    const int dir = R.dir;
    const bool unit_end = s0 + ns == nb;  // the segment holds the unit's last step
    const float lam = p.decay[bh % p.H];
    if (warp >= 4) {
        // lambda^n (n = 0..T_B), lambda^(15-n), the diagonal-block table
        // Z[m] = lambda^(m-31) for m >= 31, else 0 (m = 0..66; copy k holds
        // Z[j + k] at j, so that a 32-entry window starting anywhere can be read
        // with aligned 16-byte loads), and W buffer 0 = 0; then a barrier among
        // the 16 warps that use them
        const int t = tid - 128;
        const double l2 = log2(static_cast<double>(lam));
        for (int n = t; n <= kTB; n += kThreads - 128) pw[n] = static_cast<float>(exp2(n * l2));
        if (t < 16) murev[t] = static_cast<float>(exp2((15 - t) * l2));
        for (int idx = t; idx < 4 * 64; idx += kThreads - 128) {
            const int k = idx >> 6, j = idx & 63, m = j + k;
            float* zc = reinterpret_cast<float*>(smem_raw + L::kZ + k * L::kZstride);
            zc[j] = m >= 31 ? static_cast<float>(exp2((m - 31) * l2)) : 0.f;
        }
        for (uint32_t off = t * 16; off < 2 * L::kWsz; off += (kThreads - 128) * 16)
            st_shared_v4(sW + off, 0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
        named_barrier_sync(1, kThreads - 128);
    }
    // TMEM: S / P in two buffers (128 columns each), X in NX buffers (DC each),
    // then (DC = 64) NXI X_inter buffers, then ND dW buffers (DC = 128: the
    // fp32 state, onto which dW accumulates).
    auto tS = [&](int b) { return tmem + static_cast<uint32_t>(b * 128); };
    auto tX = [&](int b) { return tmem + 256 + static_cast<uint32_t>(b * DC); };
    auto tXI = [&](int s) {  // X_inter of step s (DC = 64)
        return tmem + 256 + static_cast<uint32_t>((Q::NX + s % (Q::NXI > 0 ? Q::NXI : 1)) * DC);
    };
    // dW (DC = 64) or the fp32 state W that dW accumulates onto (DC = 128)
    auto tD = [&](int s) {
        return tmem + 256 + static_cast<uint32_t>((Q::NX + Q::NXI) * DC + (s % Q::ND) * DC);
    };
    static_assert(256 + (Q::NX + Q::NXI + Q::ND) * DC <= static_cast<int>(kTmemCols), "TMEM columns");
    auto tile_of = [&](int step) { return dir > 0 ? s0 + step : nb - 1 - (s0 + step); };
    // fp32 state slot of segment gg of this (sequence, role)
    auto seg_slot = [&](int gg) {
        return p.seg_state + static_cast<size_t>(seg_slot_index(p, kMulti, unit, gg, nb)) * (DA * DC);
    };

    if (warp == 0) {
        // ================================================= TMA producer + MMA issuer S
        // One polling loop: a ring whose next buffer is free gets its load, and
        // S of step s = A B^T (into S buffer s % 2) is issued once A and B of
        // step s have landed and X += P C of step s-2, which read the P in that
        // buffer, is done.  Nothing here blocks, so loads never wait behind S.
        if (lane == 0 && ns > 0 && p.hold != nullptr) {
            // failure-path self-test: wait for a flag that is never set; the
            // wait runs out before any load is issued, and every role then
            // leaves through the abort flag
            const uint64_t t0 = global_ns();
            while (*reinterpret_cast<const volatile int*>(p.hold) == 0) {
                if (global_ns() - t0 > p.hold_ns) {
                    *abort_flag = 1;
                    atomicCAS(p.status, 0, kTimeoutCode | (kSiteHold << 8));
                    break;
                }
                __nanosleep(1000);
            }
        }
        if (lane == 0 && ns > 0 && !*abort_flag) {
            prefetch_tmap(&R.ta);
            prefetch_tmap(&R.tb);
            prefetch_tmap(&R.tc);
            auto load_a = [&](int s) {
                const int slot = s % Q::NA;
                const uint32_t b = bar(Q::FULL_A + slot);
                mbar_arrive_expect_tx(b, L::kAsz);
                for (int gg = 0; gg < DA / 64; ++gg)
                    load_box(sA + slot * L::kAsz + gg * 16384, &R.ta, b, gg * 64, tile_of(s) * kTB, bh, p.H, p.bthd);
            };
            // A of step s is also read by X_inter = A W, which waits for the
            // state, so its buffer comes free late; an L2 prefetch of it, made
            // when B of step s is loaded, takes the HBM latency off that load
            auto load_b = [&](int s) {
                const int slot = s % Q::NB;
                const uint32_t b = bar(Q::FULL_B + slot);
                mbar_arrive_expect_tx(b, L::kBsz);
                for (int gg = 0; gg < DA / 64; ++gg)
                    load_box(sB + slot * L::kBsz + gg * 16384, &R.tb, b, gg * 64, tile_of(s) * kTB, bh, p.H, p.bthd);
                if (s >= Q::NA)
                    for (int gg = 0; gg < DA / 64; ++gg)
                        prefetch_box(&R.ta, gg * 64, tile_of(s) * kTB, bh, p.H, p.bthd);
            };
            auto load_c = [&](int s) {
                const int slot = s % Q::NC;
                const uint32_t b = bar(Q::FULL_C + slot);
                mbar_arrive_expect_tx(b, L::kCsz);
                for (int gg = 0; gg < DC / 64; ++gg)
                    load_box(sC + slot * L::kCsz + gg * 16384, &R.tc, b, gg * 64, tile_of(s) * kTB, bh, p.H, p.bthd);
            };
            constexpr uint32_t kIdS = idesc_bf16_f32(128, kTB, 0, 0);
            const uint64_t dA0 = sdesc_sw128(sA, 16, 1024), dB0 = sdesc_sw128(sB, 16, 1024);
            auto issue_s = [&](int s) {
                const int sa = s % Q::NA, sb = s % Q::NB;
                tc_fence_after();
                const uint32_t st = tS(s & 1);
                const uint64_t da = desc_add(dA0, sa * L::kAsz), db = desc_add(dB0, sb * L::kBsz);
#pragma unroll
                for (int k = 0; k < DA / 16; ++k) {
                    const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
                    mma_bf16_ss(st, desc_add(da, off), desc_add(db, off), kIdS, k > 0);
                }
                mma_commit(bar(Q::S_DONE + (s & 1)));
                mma_commit(bar(Q::EMPTY_A + sa));
                if (Q::kTf32) mma_commit(bar(Q::EMPTY_B + sb));  // dW does not read B
            };
            // step s of a ring of n buffers may be loaded once step s - n has
            // released its buffer
            int ia = 0, ib = 0, ic = 0, is = 0;
            bool idle = false;
            uint64_t t0 = 0;
            while (is < ns || ia < ns || ib < ns || ic < ns) {
                bool prog = false;
                if (ib < ns && (ib < Q::NB ||
                                mbar_test_wait(bar(Q::EMPTY_B + ib % Q::NB), empty_par(ib, Q::NB)))) {
                    LA2_TR(3, ib);
                    load_b(ib++);
                    prog = true;
                }
                if (ia < ns && (ia < Q::NA ||
                                mbar_test_wait(bar(Q::EMPTY_A + ia % Q::NA), empty_par(ia, Q::NA)))) {
                    LA2_TR(2, ia);
                    load_a(ia++);
                    prog = true;
                }
                if (ic < ns && (ic < Q::NC ||
                                mbar_test_wait(bar(Q::EMPTY_C + ic % Q::NC), empty_par(ic, Q::NC)))) {
                    LA2_TR(4, ic);
                    load_c(ic++);
                    prog = true;
                }
                if (is < ia && is < ib &&
                    mbar_test_wait(bar(Q::FULL_A + is % Q::NA), full_par(is, Q::NA)) &&
                    mbar_test_wait(bar(Q::FULL_B + is % Q::NB), full_par(is, Q::NB)) &&
                    (is < 2 || mbar_test_wait(bar(Q::EMPTY_S + (is & 1)), empty_par(is, 2)))) {
                    LA2_TR(5, is);
                    issue_s(is);
                    LA2_TR(19, is);
                    ++is;
                    prog = true;
                }
                if (prog) {
                    idle = false;
                    continue;
                }
                if (*abort_flag) break;
                // back off briefly: this warp shares its scheduler with mask and
                // epilogue warps, which a tight polling loop would slow down
                __nanosleep(32);
                const uint64_t now = global_ns();
                if (!idle) {
                    idle = true;
                    t0 = now;
                } else if (now - t0 > 2000000000ull) {
                    *abort_flag = 1;
                    atomicCAS(p.status, 0, 5 | ((is < ns ? 20 : 10) << 8));
                    break;
                }
            }
        }
        if (lane == 0) mma_commit(bar(Q::FIN));
    } else if (warp == 1) {
        // ================================================= MMA issuer PC
        // X += P C of tile s, P read from S buffer s % 2: in bf16 mode its hi and
        // lo parts per K step of 16; in tf32 mode P is fp32, K steps of 8, with
        // the fp32 copy of C
        if (Q::kTf32 || lane == 0) {
            // d = 64: the whole warp runs the issuing loop and lane 0 issues
            // (warp-uniform descriptor arithmetic measured +4% there); d = 128:
            // lane 0 alone
            const uint32_t leader = Q::kTf32 ? lane == 0 : 1;
            constexpr uint32_t kIdX = Q::kTf32 ? idesc_tf32_f32(128, DC, 0, 0)
                                               : idesc_bf16_f32(128, DC, 0, 1);
            const uint64_t dC0 = Q::kTf32 ? sdesc_sw128(sCF, 16, 1024) : sdesc_sw128(sC, 16384, 1024);
            for (int s = 0; s < ns; ++s) {
                const int sc = Q::kTf32 ? s % Q::NCF : s % Q::NC;
                if (!wait_bar<Q::kTf32>(bar(Q::P_READY + (s & 1)), full_par(s, 2), abort_flag, p.status, 23)) break;
                if (Q::kOwnD) {
                    // X buffer s % 2 has been read out after tile s-2
                    if (s >= Q::NX && !wait_bar<Q::kTf32>(bar(Q::EMPTY_X + s % Q::NX), empty_par(s, Q::NX),
                                                abort_flag, p.status, 24))
                        break;
                } else if (!wait_bar<Q::kTf32>(bar(Q::XS + s % Q::NX), full_par(s, Q::NX), abort_flag, p.status, 24)) {
                    break;
                }
                if (Q::kTf32) {
                    if (!wait_bar<Q::kTf32>(bar(Q::CF_READY + sc), full_par(s, Q::NCF), abort_flag, p.status, 25))
                        break;
                } else if (!wait_bar<Q::kTf32>(bar(Q::FULL_C + sc), full_par(s, Q::NC), abort_flag, p.status, 25)) {
                    break;
                }
                LA2_TR(6, s);
                tc_fence_after();
                const uint32_t xt = tX(s % Q::NX), st = tS(s & 1);
                if constexpr (Q::kTf32) {
                    const uint64_t dc = desc_add(dC0, sc * L::kCFsz);
#pragma unroll 4
                    for (int k = 0; k < kTB / 8; ++k)
                        mma_tf32_ts_w(xt, st + k * 8, desc_add(dc, (k >> 2) * (DC * 128) + (k & 3) * 32),
                                    kIdX, Q::kOwnD ? (k > 0) : 1, leader);
                } else {
                    const uint64_t dc = desc_add(dC0, sc * L::kCsz);
#pragma unroll
                    for (int k = 0; k < kTB / 16; ++k) {
                        const uint64_t cdesc = desc_add(dc, k * 2048);
                        mma_bf16_ts_w(xt, st + k * 16, cdesc, kIdX, Q::kOwnD ? (k > 0) : 1, leader);
                        mma_bf16_ts_w(xt, st + k * 16 + 8, cdesc, kIdX, 1, leader);
                    }
                }
                mma_commit_w(bar(Q::PC_DONE + s % Q::NX), leader);
                mma_commit_w(bar(Q::EMPTY_S + (s & 1)), leader);
                mma_commit_w(bar((Q::kTf32 ? Q::EMPTY_CF : Q::EMPTY_C) + sc), leader);
                LA2_TR(20, s);
            }
            mma_commit_w(bar(Q::FIN), leader);
        }
    } else if (warp == 2) {
        // ================================================= MMA issuer XW
        // X = A hi(W) + A lo(W) into X buffer s % 2
        if (Q::kTf32 || lane == 0) {
            const uint32_t leader = Q::kTf32 ? lane == 0 : 1;
            constexpr uint32_t kIdX = idesc_bf16_f32(128, DC, 0, 1);
            const uint64_t dA0 = sdesc_sw128(sA, 16, 1024), dW0 = sdesc_sw128(sW, DA * 128, 1024);
            for (int s = 0; s < ns; ++s) {
                const int sa = s % Q::NA, sw = s % Q::NW;
                // W_READY completes once the epilogue has set W of this step (the
                // initial state, or the update after the previous tile, which has
                // also read the dW that sat in this X buffer)
                if (!wait_bar<Q::kTf32>(bar(Q::W_READY + sw), full_par(s, Q::NW), abort_flag, p.status, 30)) break;
                if (!wait_bar<Q::kTf32>(bar(Q::FULL_A + sa), full_par(s, Q::NA), abort_flag, p.status, 31)) break;
                if constexpr (Q::kOwnD) {
                    // X_inter buffer s % 2 has been read out after tile s-2
                    if (s >= Q::NXI && !wait_bar<Q::kTf32>(bar(Q::EMPTY_XI + s % Q::NXI), empty_par(s, Q::NXI),
                                                           abort_flag, p.status, 32))
                        break;
                } else if (s >= Q::NX && !wait_bar<Q::kTf32>(bar(Q::EMPTY_X + s % Q::NX), empty_par(s, Q::NX),
                                                   abort_flag, p.status, 32)) {
                    break;
                }
                LA2_TR(7, s);
                tc_fence_after();
                const uint32_t xt = Q::kOwnD ? tXI(s) : tX(s % Q::NX);
                const uint64_t da = desc_add(dA0, sa * L::kAsz), dw = desc_add(dW0, sw * 2 * L::kWsz);
#pragma unroll
                for (int k = 0; k < DA / 16; ++k) {
                    const uint64_t adesc = desc_add(da, (k >> 2) * 16384 + (k & 3) * 32);
                    mma_bf16_ss_w(xt, adesc, desc_add(dw, k * 2048), kIdX, k > 0, leader);
                    mma_bf16_ss_w(xt, adesc, desc_add(dw, L::kWsz + k * 2048), kIdX, 1, leader);
                }
                mma_commit_w(bar(Q::XW_DONE + s % Q::NXW), leader);
                mma_commit_w(bar(Q::EMPTY_A + sa), leader);
                mma_commit_w(bar(Q::EMPTY_W + sw), leader);
                LA2_TR(21, s);
            }
            mma_commit_w(bar(Q::FIN), leader);
        }
    } else if (warp == 3) {
        // ================================================= MMA issuer dW
        // dW = (w_s B)^T C of tile s: bf16 mode hi(w_s B)^T C + lo(w_s B)^T C,
        // tf32 mode the fp32 copies of w_s B and C
        if (Q::kTf32 || lane == 0) {
            const uint32_t leader = Q::kTf32 ? lane == 0 : 1;
            constexpr uint32_t kIdW = Q::kTf32 ? idesc_tf32_f32(DA, DC, 0, 0) : idesc_bf16_f32(DA, DC, 1, 1);
            const uint64_t dB0 = Q::kTf32 ? sdesc_sw128(sWB, 16, 1024) : sdesc_sw128(sB, 16384, 1024);
            const uint64_t dL0 = sdesc_sw128(sBlo, 16384, 1024);
            const uint64_t dC0 = Q::kTf32 ? sdesc_sw128(sCF, 16, 1024) : sdesc_sw128(sC, 16384, 1024);
            for (int s = 0; s < ns; ++s) {
                const int sb = Q::kTf32 ? s % Q::NWB : s % Q::NB;
                const int sc = Q::kTf32 ? s % Q::NCF : s % Q::NC;
                const int sl = Q::kTf32 ? 0 : s % Q::NBLO;
                if (Q::kTf32) {
                    if (!wait_bar<Q::kTf32>(bar(Q::WB_READY + sb), full_par(s, Q::NWB), abort_flag, p.status, 33)) break;
                    if (!wait_bar<Q::kTf32>(bar(Q::CF_READY + sc), full_par(s, Q::NCF), abort_flag, p.status, 34)) break;
                } else {
                    if (!wait_bar<Q::kTf32>(bar(Q::BS + sb), full_par(s, Q::NB), abort_flag, p.status, 33)) break;
                    if (!wait_bar<Q::kTf32>(bar(Q::FULL_C + sc), full_par(s, Q::NC), abort_flag, p.status, 34)) break;
                }
                if constexpr (Q::kWT) {
                    // the state holds lambda(s) W_s: written by the epilogue's set-up
                    // (s = 0) or by the update after tile s-1
                    if (!wait_bar<Q::kTf32>(bar(Q::EMPTY_D), full_par(s, 1), abort_flag, p.status, 36)) break;
                } else if (s >= Q::ND && !wait_bar<Q::kTf32>(bar(Q::EMPTY_D + s % Q::ND), empty_par(s, Q::ND),
                                                             abort_flag, p.status, 35)) {
                    // the update after tile s - ND has read this dW buffer
                    break;
                }
                LA2_TR(8, s);
                tc_fence_after();
                const uint32_t dt = tD(s);
                if constexpr (Q::kTf32) {
                    const uint64_t db = desc_add(dB0, sb * L::kWBsz), dc = desc_add(dC0, sc * L::kCFsz);
#pragma unroll 4
                    for (int k = 0; k < kTB / 8; ++k)
                        mma_tf32_ss_w(dt, desc_add(db, (k >> 2) * (DA * 128) + (k & 3) * 32),
                                    desc_add(dc, (k >> 2) * (DC * 128) + (k & 3) * 32), kIdW, k > 0, leader);
                    mma_commit_w(bar(Q::D_DONE + (s % Q::ND)), leader);
                    mma_commit_w(bar(Q::EMPTY_WB + sb), leader);
                    mma_commit_w(bar(Q::EMPTY_CF + sc), leader);
                } else {
                    const uint64_t db = desc_add(dB0, sb * L::kBsz), dl = desc_add(dL0, sl * L::kBsz);
                    const uint64_t dc = desc_add(dC0, sc * L::kCsz);
#pragma unroll
                    for (int k = 0; k < kTB / 16; ++k) {
                        const uint64_t cdesc = desc_add(dc, k * 2048);
                        mma_bf16_ss_w(dt, desc_add(db, k * 2048), cdesc, kIdW, (Q::kWT || k > 0) ? 1u : 0u, leader);
                        mma_bf16_ss_w(dt, desc_add(dl, k * 2048), cdesc, kIdW, 1, leader);
                    }
                    mma_commit_w(bar(Q::D_DONE + (s % Q::ND)), leader);
                    mma_commit_w(bar(Q::EMPTY_B + sb), leader);
                    mma_commit_w(bar(Q::EMPTY_BLO + sl), leader);
                    mma_commit_w(bar(Q::EMPTY_C + sc), leader);
                }
                LA2_TR(22, s);
            }
            mma_commit_w(bar(Q::FIN), leader);
        }
    } else if (warp >= 4 && warp < 12) {
        // ================================================= mask group
        // two warps per lane quadrant; part p of a quadrant takes half the work
        const int quad = warp & 3, part = (warp - 4) >> 2;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const float ws = dir > 0 ? pw[kTB - 1 - r] : pw[r];
        // diagonal 32 x 32 block of this quadrant: row `lane` reads a 32-entry
        // window of Z (dir > 0: weight of column j = Z[lane - j + 31]; dir < 0:
        // Z[j - lane + 31]), from the copy that makes the window 16-byte aligned
        const int zs = dir > 0 ? lane : 31 - lane;
        const uint32_t zwin = base + L::kZ + (zs & 3) * L::kZstride + (zs - (zs & 3)) * 4;
        const float* mu = dir > 0 ? murev : pw;
        // The last tile of a forward scan may hold n < T_B rows: its state
        // update then uses lambda^(n-1-r) (and lambda^n for the old state), so
        // that the state after it is the state after position T-1 exactly.  No
        // output reads that state; only the final state does.
        const int nlast = T - (nb - 1) * kTB;
        const float ws_last = r < nlast ? pw[max(nlast - 1 - r, 0)] : 0.f;
        // the per-position factor of this thread's row of the tile of step s
        const float* colf = (kNorm && R.colf) ? R.colf + static_cast<size_t>(bh) * T : nullptr;
        auto f_of = [&](int s, int row) -> float {
            const int t = tile_of(s) * kTB + row;
            return t < T ? __ldg(colf + t) : 0.f;
        };
        auto ws_of = [&](int s) {
            const float w = (dir > 0 && unit_end && s == ns - 1) ? ws_last : ws;
            if constexpr (kNorm) return colf ? w * f_of(s, r) : w;
            return w;
        };
        // P's columns times the factors of their positions (32 columns of block pr)
        auto colscale = [&](int s, int pr, float (&sv)[32]) {
            if constexpr (!kNorm) return;
            if (colf == nullptr) return;
#pragma unroll
            for (int u = 0; u < 32; ++u) sv[u] *= f_of(s, 32 * pr + u);
        };
        // P = S * lambda^|r-c| on the causal side, 0 elsewhere, 32 columns (one
        // pair of K = 16 groups) at a time.  pr == quad is the diagonal block;
        // whole pairs on the causal side use lambda^|r-c| = alpha mu(c), with
        // alpha = lambda^(r - 16 grp - 15) resp. lambda^(16 grp - r), exponents
        // in [1, 127], and mu = lambda^(15-u) resp. lambda^u.  Every S column
        // is loaded before it is overwritten, also columns the mask zeroes:
        // storing over S columns that were not read first made the following
        // TMEM-operand MMAs about 10x slower.
        auto weigh = [&](int pr, float (&sv)[32]) {
            const bool diag = pr == quad;
            const bool causal = (dir > 0) == (pr < quad);
            if (diag) {
#pragma unroll
                for (int t4 = 0; t4 < 8; ++t4) {
                    float z[4];
                    ld_shared_v4f(zwin + 16 * t4, z);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int t = 4 * t4 + e;           // window index
                        const int j = dir > 0 ? 31 - t : t;  // column in the block
                        sv[j] *= z[e];
                    }
                }
            } else if (causal) {
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int grp = 2 * pr + h2;
                    const float alpha = pw[dir > 0 ? r - 16 * grp - 15 : 16 * grp - r];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float2 m = *reinterpret_cast<const float2*>(mu + 2 * u);
                        const float2 w = mul2(m, make_float2(alpha, alpha));
                        const float2 pv = mul2(make_float2(sv[16 * h2 + 2 * u], sv[16 * h2 + 2 * u + 1]), w);
                        sv[16 * h2 + 2 * u] = pv.x;
                        sv[16 * h2 + 2 * u + 1] = pv.y;
                    }
                }
            } else {
#pragma unroll
                for (int u = 0; u < 32; ++u) sv[u] = 0.f;
            }
        };
        // tf32 mode: transposed stores go to row n = 32 part + 8 k + j, word
        // `lane` of a 128-byte row; the part of the swizzled address that depends
        // on j and the lane is fixed per thread, the rest ((4 part + k) * 1024) is
        // an immediate
        uint32_t toff[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            toff[j] = static_cast<uint32_t>(part * 4096 + j * 128 + (((lane >> 2) ^ j) << 4) + (lane & 3) * 4);
        for (int s = 0; s < ns; ++s) {
            if constexpr (Q::kTf32) {
                // C -> fp32 C^T (the K-major tf32 B operand of X += P C and dW): row r
                // of C, columns 32 part .. 32 part + 31 (bf16 chunks 4 part + k), each
                // to word r of row n of C^T; the lanes of a warp (consecutive r) fill
                // one whole 128-byte row, so the scalar stores meet no bank conflict
                const int sc = s % Q::NC, scf = s % Q::NCF;
                if (!wait_bar<Q::kTf32>(bar(Q::FULL_C + sc), full_par(s, Q::NC), abort_flag, p.status, 42)) break;
                if (s >= Q::NCF && !wait_bar<Q::kTf32>(bar(Q::EMPTY_CF + scf), empty_par(s, Q::NCF), abort_flag,
                                             p.status, 43))
                    break;
                {
                    const uint32_t src = sC + sc * L::kCsz, dst = sCF + scf * L::kCFsz + quad * (DC * 128);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint32_t v[4];
                        ld_shared_v4(src + sw128(r, 4 * part + k), v[0], v[1], v[2], v[3]);
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            st_shared_f32(dst + toff[2 * u] + k * 1024, bf16lo_to_f32(v[u]));
                            st_shared_f32(dst + toff[2 * u + 1] + k * 1024, bf16hi_to_f32(v[u]));
                        }
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(bar(Q::EMPTY_C + sc));
                mbar_arrive(bar(Q::CF_READY + scf));
                // w_s B -> fp32 (w_s B)^T (the K-major tf32 A operand of dW), laid out
                // like C^T; B itself is left for S
                const int sb = s % Q::NB, swb = s % Q::NWB;
                if (!wait_bar<Q::kTf32>(bar(Q::FULL_B + sb), full_par(s, Q::NB), abort_flag, p.status, 44)) break;
                if (s >= Q::NWB && !wait_bar<Q::kTf32>(bar(Q::EMPTY_WB + swb), empty_par(s, Q::NWB), abort_flag,
                                             p.status, 45))
                    break;
                {
                    const float ws_s = ws_of(s);
                    const uint32_t src = sB + sb * L::kBsz, dst = sWB + swb * L::kWBsz + quad * (DA * 128);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint32_t v[4];
                        ld_shared_v4(src + sw128(r, 4 * part + k), v[0], v[1], v[2], v[3]);
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float2 w = mul2(make_float2(bf16lo_to_f32(v[u]), bf16hi_to_f32(v[u])),
                                                  make_float2(ws_s, ws_s));
                            st_shared_f32(dst + toff[2 * u] + k * 1024, w.x);
                            st_shared_f32(dst + toff[2 * u + 1] + k * 1024, w.y);
                        }
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(bar(Q::EMPTY_B + sb));
                mbar_arrive(bar(Q::WB_READY + swb));
                if (tid == 128) LA2_TR(10, s);
                // P in place, fp32
                if (!wait_bar<Q::kTf32>(bar(Q::S_DONE + (s & 1)), full_par(s, 2), abort_flag, p.status, 40)) break;
                if (tid == 128) LA2_TR(9, s);
                tc_fence_after();
                const uint32_t st = tS(s & 1);
#pragma unroll 1
                for (int pr = part; pr < kTB / 32; pr += 2) {
                    float sv[32];
                    tmem_ld32(st + lane_off + pr * 32, sv);
                    weigh(pr, sv);
                    colscale(s, pr, sv);
                    tmem_st32(st + lane_off + pr * 32, sv);
                }
            } else {
                if (!wait_bar<Q::kTf32>(bar(Q::S_DONE + (s & 1)), full_par(s, 2), abort_flag, p.status, 40)) break;
                if (tid == 128) LA2_TR(9, s);
                const uint32_t st = tS(s & 1);
                tc_fence_after();
                // row r of w_s B (S, which reads B unscaled, is done): hi in place,
                // lo into its own buffer once the dW that last read that buffer is
                // done.  Part p does the chunks of half p of the row.
                const int sl = s % Q::NBLO;
                if (s >= Q::NBLO && !wait_bar<Q::kTf32>(bar(Q::EMPTY_BLO + sl), empty_par(s, Q::NBLO), abort_flag,
                                              p.status, 41))
                    break;
                const uint32_t sBs = sB + (s % Q::NB) * L::kBsz, sBl = sBlo + sl * L::kBsz;
                const float ws_s = ws_of(s);
#pragma unroll
                for (int k = 0; k < DA / 16; ++k) {
                    const int chunk = part * (DA / 16) + k;
                    const uint32_t off = (chunk >> 3) * 16384 + sw128(r, chunk & 7);
                    uint32_t v[4], h[4], l[4];
                    ld_shared_v4(sBs + off, v[0], v[1], v[2], v[3]);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        split_pack2v(mul2(make_float2(bf16lo_to_f32(v[u]), bf16hi_to_f32(v[u])),
                                          make_float2(ws_s, ws_s)),
                                     h[u], l[u]);
                    st_shared_v4(sBs + off, h[0], h[1], h[2], h[3]);
                    st_shared_v4(sBl + off, l[0], l[1], l[2], l[3]);
                }
                fence_proxy_async_smem();
                mbar_arrive(bar(Q::BS + (s % Q::NB)));
                if (tid == 128) LA2_TR(10, s);
                // P as hi + lo bf16, over the 16 columns of S each group of 16 came
                // from: [hi (8 cols) | lo (8 cols)], the A-operand layout of one
                // K = 16 step
#pragma unroll 1
                for (int pr = part; pr < kTB / 32; pr += 2) {
                    float sv[32];
                    tmem_ld32(st + lane_off + pr * 32, sv);
                    weigh(pr, sv);
                    colscale(s, pr, sv);
                    uint32_t pk[32];
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            split_pack2v(make_float2(sv[16 * h2 + 2 * u], sv[16 * h2 + 2 * u + 1]),
                                         pk[16 * h2 + u], pk[16 * h2 + 8 + u]);
                    tmem_st32u(st + lane_off + pr * 32, pk);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(Q::P_READY + (s & 1)));
            if (tid == 128) LA2_TR(11, s);
        }
    } else if (warp >= 12 && warp < 20) {
        // ================================================= epilogue group
        const int quad = warp & 3, half = (warp - 12) >> 2;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        constexpr int kCols = DC / 2;                 // columns of X and W this thread handles
        const int c0 = half * kCols;
        const float wx = dir > 0 ? pw[r + 1] : pw[kTB - r];
        const float lamTB = pw[kTB];
        // The reverse scan's first tile (the sequence's last, n = nlast rows)
        // takes a given state as entering at position T-1: its rows weigh it
        // by lambda^(n-1-r) and it decays by lambda^(n-1) across the tile.
        const int nlast = T - (nb - 1) * kTB;
        const bool first_rev = dir < 0 && s0 == 0;
        const float wx_first = r < nlast ? pw[nlast - 1 - r] : 0.f;
        const bool owns_w_row = (DA == 128) || (lane < 16);
        const int wrow = (DA == 128) ? r : quad * 16 + (lane & 15);
        // With 32 columns per thread (DC = 64) each owner thread keeps its part
        // of the state in fp32 registers; the hi/lo pair in shared memory is
        // then written, never read back.
        constexpr bool kWReg = kCols == 32;
        float wreg[kWReg ? 32 : 1];
#pragma unroll
        for (int u = 0; u < (kWReg ? 32 : 1); ++u) wreg[u] = 0.f;
        // initial state of this segment, W_in(j) = f_{j-1} W_in(j-1) + S_{j-1}
        // with f_i = lambda^(T_B n_i) (n_i tiles in segment i: L, except for
        // segment 0, which ends at step L - ph) and W_in(0) the given initial
        // state (or 0), as its hi/lo bf16 pair in W buffer 0
        // the state's old-value factor before the dW of step s: lambda^T_B,
        // lambda^n for the forward scan's last (n-row) tile, lambda^(n-1) for the
        // reverse scan's first tile (an entering state at position T-1)
        const bool has_last = dir > 0 && unit_end;
        auto lam_of = [&](int s) -> float {
            return (has_last && s == ns - 1) ? pw[nlast] : ((first_rev && s == 0) ? pw[nlast - 1] : lamTB);
        };
        {
            const bool mine = (sj > 0 || R.init != nullptr) && owns_w_row;
            const double l2 = log2(static_cast<double>(lam));
            const float fL = static_cast<float>(exp2(static_cast<double>(kTB) * p.seg_tiles * l2));
            // segment 0 has n0 tiles; in the reverse direction its first tile
            // decays an entering state by lambda^(nlast-1) instead of lambda^T_B
            const int n0 = p.seg_tiles - seg_phase(p, kMulti, unit, nb);
            const double e0 = dir > 0 ? static_cast<double>(kTB) * n0
                                      : static_cast<double>(kTB) * (n0 - 1) + (nlast - 1);
            const float f0 = static_cast<float>(exp2(e0 * l2));
            const float* w0 = R.init ? R.init + static_cast<size_t>(bh) * (DA * DC) : nullptr;
            // DC = 128: the fp32 state in TMEM starts as lambda(0) W_in, so that dW
            // of step 0 accumulates onto it (every lane stores; rows a thread
            // does not own are 0)
            const float f0s = lam_of(0);
            float wt[Q::kWT ? 32 : 1];
#pragma unroll
            for (int k = 0; k < kCols / 16; ++k) {
                const uint32_t col = c0 + k * 16;
                float w[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) w[u] = 0.f;
                if (mine) {
                    if (w0 && R.init_t) {
#pragma unroll
                        for (int u = 0; u < 16; ++u) w[u] = w0[static_cast<size_t>(col + u) * DA + wrow];
                    } else if (w0) {
#pragma unroll
                        for (int u = 0; u < 16; ++u) w[u] = w0[static_cast<size_t>(wrow) * DC + col + u];
                    }
                    for (int gp = 0; gp < sj; ++gp) {
                        const float f = gp == 0 ? f0 : fL;
                        const float* src = seg_slot(gp) + static_cast<size_t>(wrow) * DC + col;
#pragma unroll
                        for (int u = 0; u < 16; ++u) w[u] = fmaf(f, w[u], src[u]);
                    }
                    if constexpr (kWReg) {
#pragma unroll
                        for (int u = 0; u < 16; ++u) wreg[16 * (k & 1) + u] = w[u];
                    }
                    const uint32_t grpo = (col >> 6) * (DA * 128);
                    const int q = (col & 63) >> 3;
                    uint32_t h[8], l[8];
#pragma unroll
                    for (int z = 0; z < 8; ++z) split_pack2(w[2 * z], w[2 * z + 1], h[z], l[z]);
                    st_shared_v4(sW + grpo + sw128(wrow, q), h[0], h[1], h[2], h[3]);
                    st_shared_v4(sW + grpo + sw128(wrow, q + 1), h[4], h[5], h[6], h[7]);
                    st_shared_v4(sW + L::kWsz + grpo + sw128(wrow, q), l[0], l[1], l[2], l[3]);
                    st_shared_v4(sW + L::kWsz + grpo + sw128(wrow, q + 1), l[4], l[5], l[6], l[7]);
                }
                if constexpr (Q::kWT) {
#pragma unroll
                    for (int u = 0; u < 16; ++u) wt[16 * (k & 1) + u] = f0s * w[u];
                    if (k & 1) tmem_st32(tD(0) + lane_off + col - 16, wt);
                }
            }
            if constexpr (Q::kWT) {
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(Q::EMPTY_D));
            }
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(Q::W_READY + 0));
        // output rows: [B, H, T, DC] (row stride DC) or [B, T, H, DC] (stride H DC)
        const size_t xrs = p.bthd ? static_cast<size_t>(p.H) * DC : static_cast<size_t>(DC);
        const size_t xoff = p.bthd ? (static_cast<size_t>(bh / p.H) * T * p.H + bh % p.H) * DC
                                   : static_cast<size_t>(bh) * T * DC;
        char* const xg = static_cast<char*>(R.x) + xoff * (kXb16 ? 2 : 4);

        // X row r *= w_x(r) (the inter-tile term, still alone in X)
        auto scale = [&](int s) -> bool {
            if (!wait_bar<Q::kTf32>(bar(Q::XW_DONE + s % Q::NXW), full_par(s, Q::NXW), abort_flag, p.status, 50))
                return false;
            if (tid == 384) LA2_TR(14, s);
            tc_fence_after();
            const uint32_t xt = tX(s % Q::NX);
            const float wxs = (first_rev && s == 0) ? wx_first : wx;
#pragma unroll 1
            for (int k = 0; k < kCols / 32; ++k) {
                float x[32];
                const uint32_t col = c0 + k * 32;
                tmem_ld32(xt + lane_off + col, x);
#pragma unroll
                for (int u = 0; u < 32; ++u) x[u] *= wxs;
                tmem_st32(xt + lane_off + col, x);
            }
            tmem_wait_st();
            tc_fence_before();
            if constexpr (Q::NXS > 0) mbar_arrive(bar(Q::XS + s % Q::NXS));
            if (tid == 384) LA2_TR(15, s);
            return true;
        };
        // W <- lambda^T_B W + dW, from W buffer s % NW into (s+1) % NW.  The
        // state is kept as its hi + lo bf16 pair (a 16-bit significand, ~2^-17
        // relative per update), which is also the next tile's MMA operand.
        auto update = [&](int s) -> bool {
            const float lam_s = lam_of(s);
            if (!wait_bar<Q::kTf32>(bar(Q::D_DONE + (s % Q::ND)), full_par(s, Q::ND), abort_flag, p.status, 51))
                return false;
            // the X MMA that last read the W buffer written here is done
            if (s + 1 >= Q::NW && !wait_bar<Q::kTf32>(bar(Q::EMPTY_W + (s + 1) % Q::NW),
                                            full_par(s + 1 - Q::NW, Q::NW), abort_flag, p.status, 52))
                return false;
            if (tid == 384) LA2_TR(12, s);
            tc_fence_after();
            const uint32_t wsrc = sW + (s % Q::NW) * 2 * L::kWsz;
            const uint32_t wdst = sW + ((s + 1) % Q::NW) * 2 * L::kWsz;
            const uint32_t dt = tD(s);
            if constexpr (Q::kWT) {
                // W_{s+1} = lambda(s) W_s + dW_s, accumulated in fp32 in TMEM: its
                // hi/lo pair to the next A W's buffer, the final state from it,
                // and lambda(s+1) W_{s+1} written back for the next dW
                const bool more = s + 1 < ns;
                const float lam_n = more ? lam_of(s + 1) : 1.f;
                const bool fin_now = unit_end && s == ns - 1 && R.fin != nullptr && owns_w_row;
                float* const fin = R.fin ? R.fin + static_cast<size_t>(bh) * (DA * DC) + static_cast<size_t>(wrow) * DC
                                         : nullptr;
                const float fs = dir > 0 ? 1.f : lam;
#pragma unroll 1
                for (int k = 0; k < kCols / 32; ++k) {
                    float w[32];
                    tmem_ld32(dt + lane_off + c0 + k * 32, w);
                    if (owns_w_row) {
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const uint32_t col = c0 + k * 32 + hh * 16;
                            const uint32_t o0 = (col >> 6) * (DA * 128) + sw128(wrow, (col & 63) >> 3);
                            const uint32_t o1 = (col >> 6) * (DA * 128) + sw128(wrow, ((col & 63) >> 3) + 1);
                            uint32_t h[8], l[8];
#pragma unroll
                            for (int z = 0; z < 8; ++z)
                                split_pack2v(make_float2(w[16 * hh + 2 * z], w[16 * hh + 2 * z + 1]), h[z], l[z]);
                            st_shared_v4(wdst + o0, h[0], h[1], h[2], h[3]);
                            st_shared_v4(wdst + o1, h[4], h[5], h[6], h[7]);
                            st_shared_v4(wdst + L::kWsz + o0, l[0], l[1], l[2], l[3]);
                            st_shared_v4(wdst + L::kWsz + o1, l[4], l[5], l[6], l[7]);
                        }
                    }
                    if (fin_now) {
                        // the final state in fp32; a reverse scan hands on lambda
                        // times its state at position 0
#pragma unroll
                        for (int u = 0; u < 32; ++u) fin[c0 + k * 32 + u] = fs * w[u];
                    }
                    if (more) {
#pragma unroll
                        for (int u = 0; u < 32; ++u) w[u] *= lam_n;
                        tmem_st32(dt + lane_off + c0 + k * 32, w);
                    }
                }
                if (more) tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(Q::EMPTY_D));
            }
#pragma unroll 1
            for (int k = 0; k < (Q::kWT ? 0 : kCols / 32); ++k) {
                float d[32];
                tmem_ld32(dt + lane_off + c0 + k * 32, d);
                if (tid == 384 && k == 0) LA2_TR(23, s);
                if (Q::kOwnD && k == kCols / 32 - 1) {
                    tc_fence_before();
                    mbar_arrive(bar(Q::EMPTY_D + s % Q::ND));
                }
                if (kWReg && owns_w_row) {
                    const float2 lam2 = make_float2(lam_s, lam_s);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const uint32_t col = c0 + hh * 16;
                        const uint32_t o0 = (col >> 6) * (DA * 128) + sw128(wrow, (col & 63) >> 3);
                        const uint32_t o1 = (col >> 6) * (DA * 128) + sw128(wrow, ((col & 63) >> 3) + 1);
                        uint32_t h[8], l[8];
#pragma unroll
                        for (int z = 0; z < 8; ++z) {
                            const int u = 16 * hh + 2 * z;
                            const float2 w = fma2(lam2, make_float2(wreg[u], wreg[u + 1]),
                                                  make_float2(d[u], d[u + 1]));
                            wreg[u] = w.x;
                            wreg[u + 1] = w.y;
                            split_pack2v(w, h[z], l[z]);
                        }
                        st_shared_v4(wdst + o0, h[0], h[1], h[2], h[3]);
                        st_shared_v4(wdst + o1, h[4], h[5], h[6], h[7]);
                        st_shared_v4(wdst + L::kWsz + o0, l[0], l[1], l[2], l[3]);
                        st_shared_v4(wdst + L::kWsz + o1, l[4], l[5], l[6], l[7]);
                    }
                } else if (owns_w_row) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const uint32_t col = c0 + k * 32 + hh * 16;
                        const uint32_t o0 = (col >> 6) * (DA * 128) + sw128(wrow, (col & 63) >> 3);
                        const uint32_t o1 = (col >> 6) * (DA * 128) + sw128(wrow, ((col & 63) >> 3) + 1);
                        uint32_t h[8], l[8];
                        ld_shared_v4(wsrc + o0, h[0], h[1], h[2], h[3]);
                        ld_shared_v4(wsrc + o1, h[4], h[5], h[6], h[7]);
                        ld_shared_v4(wsrc + L::kWsz + o0, l[0], l[1], l[2], l[3]);
                        ld_shared_v4(wsrc + L::kWsz + o1, l[4], l[5], l[6], l[7]);
#pragma unroll
                        for (int z = 0; z < 8; ++z) {
                            const float w0 = fmaf(lam_s, bf16lo_to_f32(h[z]) + bf16lo_to_f32(l[z]),
                                                  d[16 * hh + 2 * z]);
                            const float w1 = fmaf(lam_s, bf16hi_to_f32(h[z]) + bf16hi_to_f32(l[z]),
                                                  d[16 * hh + 2 * z + 1]);
                            split_pack2(w0, w1, h[z], l[z]);
                        }
                        st_shared_v4(wdst + o0, h[0], h[1], h[2], h[3]);
                        st_shared_v4(wdst + o1, h[4], h[5], h[6], h[7]);
                        st_shared_v4(wdst + L::kWsz + o0, l[0], l[1], l[2], l[3]);
                        st_shared_v4(wdst + L::kWsz + o1, l[4], l[5], l[6], l[7]);
                    }
                }
            }
            if (!Q::kWT && unit_end && s == ns - 1 && R.fin && owns_w_row) {
                // the final state: fp32 from registers (32 columns per thread;
                // DC = 128 wrote it above from TMEM); a reverse scan hands on
                // lambda times its state at position 0
                float* fin = R.fin + static_cast<size_t>(bh) * (DA * DC) + static_cast<size_t>(wrow) * DC;
                const float fs = dir > 0 ? 1.f : lam;
                if constexpr (kWReg) {
#pragma unroll
                    for (int u = 0; u < 32; ++u) fin[c0 + u] = fs * wreg[u];
                } else {
#pragma unroll 1
                    for (int cc = 0; cc < kCols; cc += 8) {
                        const uint32_t col = c0 + cc;
                        const uint32_t o = (col >> 6) * (DA * 128) + sw128(wrow, (col & 63) >> 3);
                        uint32_t h[4], l[4];
                        ld_shared_v4(wdst + o, h[0], h[1], h[2], h[3]);
                        ld_shared_v4(wdst + L::kWsz + o, l[0], l[1], l[2], l[3]);
#pragma unroll
                        for (int z = 0; z < 4; ++z) {
                            fin[col + 2 * z] = fs * (bf16lo_to_f32(h[z]) + bf16lo_to_f32(l[z]));
                            fin[col + 2 * z + 1] = fs * (bf16hi_to_f32(h[z]) + bf16hi_to_f32(l[z]));
                        }
                    }
                }
            }
            if (tid == 384) LA2_TR(24, s);
            fence_proxy_async_smem();
            if (tid == 384) LA2_TR(25, s);
            tc_fence_before();
            mbar_arrive(bar(Q::W_READY + (s + 1) % Q::NW));
            if (tid == 384) LA2_TR(13, s);
            return true;
        };
        // X of tile s, 32 columns at a time, read with the 16x256b TMEM shape:
        // each group of four lanes then holds 8 consecutive floats of one row,
        // so every float2 store of a warp fills whole 32-byte sectors (eight
        // rows per instruction).  The X buffer is released once read.
        auto output = [&](int s) -> bool {
            if (!wait_bar<Q::kTf32>(bar(Q::PC_DONE + s % Q::NX), full_par(s, Q::NX), abort_flag, p.status, 53))
                return false;
            if (Q::kOwnD &&
                !wait_bar<Q::kTf32>(bar(Q::XW_DONE + s % Q::NXW), full_par(s, Q::NXW), abort_flag, p.status, 54))
                return false;
            if (tid == 384) LA2_TR(16, s);
            tc_fence_after();
            const int i = tile_of(s);
            const uint32_t xt = tX(s % Q::NX);
            const int t4 = lane >> 2, tm = lane & 3;
            const uint32_t l0 = static_cast<uint32_t>(quad * 32) << 16;
            const uint32_t l1 = static_cast<uint32_t>(quad * 32 + 16) << 16;
            // w_x of the four rows this thread holds (lane halves lh, rows +0 / +8)
            float wxr[4];
            if constexpr (Q::kOwnD) {
#pragma unroll
                for (int lh = 0; lh < 2; ++lh)
#pragma unroll
                    for (int h8 = 0; h8 < 2; ++h8) {
                        const int rr = quad * 32 + lh * 16 + t4 + 8 * h8;
                        wxr[2 * lh + h8] = (first_rev && s == 0)
                                               ? (rr < nlast ? pw[nlast - 1 - rr] : 0.f)
                                               : (dir > 0 ? pw[rr + 1] : pw[kTB - rr]);
                    }
            }
#pragma unroll 1
            for (int b = 0; b < kCols / 32; ++b) {
                float v[32];
                const uint32_t col = c0 + 32 * b;
                tmem_ld16x256b_x4_pair(xt + l0 + col, xt + l1 + col, v);
                if constexpr (Q::kOwnD) {
                    float vi[32];
                    tmem_ld16x256b_x4_pair(tXI(s) + l0 + col, tXI(s) + l1 + col, vi);
#pragma unroll
                    for (int lh = 0; lh < 2; ++lh)
#pragma unroll
                        for (int j = 0; j < 4; ++j)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int idx = 16 * lh + 4 * j + e;
                                v[idx] = fmaf(wxr[2 * lh + (e >> 1)], vi[idx], v[idx]);
                            }
                }
                if (b == kCols / 32 - 1) {
                    tc_fence_before();
                    mbar_arrive(bar(Q::EMPTY_X + s % Q::NX));
                    if constexpr (Q::NXI > 0) mbar_arrive(bar(Q::EMPTY_XI + s % Q::NXI));
                }
                if constexpr (kXb16) {
                    // one bf16 pair per store: a warp writes 16 bytes of each of 8 rows
#pragma unroll
                    for (int lh = 0; lh < 2; ++lh) {
                        const int row = i * kTB + quad * 32 + lh * 16 + t4;
                        uint16_t* const x0 = reinterpret_cast<uint16_t*>(xg) + static_cast<size_t>(row) * xrs;
                        uint16_t* const x8 = x0 + 8 * xrs;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int cc = static_cast<int>(col) + 8 * j + 2 * tm;
                            if (row < T)
                                st_global_b32(x0 + cc, pack_bf16x2(v[16 * lh + 4 * j], v[16 * lh + 4 * j + 1]));
                            if (row + 8 < T)
                                st_global_b32(x8 + cc,
                                              pack_bf16x2(v[16 * lh + 4 * j + 2], v[16 * lh + 4 * j + 3]));
                        }
                    }
                } else {
                    float* const xf = reinterpret_cast<float*>(xg);
#pragma unroll
                    for (int lh = 0; lh < 2; ++lh) {
                        const int row = i * kTB + quad * 32 + lh * 16 + t4;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int cc = static_cast<int>(col) + 8 * j + 2 * tm;
                            if (row < T)
                                st_global_v2(xf + static_cast<size_t>(row) * xrs + cc, v[16 * lh + 4 * j],
                                             v[16 * lh + 4 * j + 1]);
                            if (row + 8 < T)
                                st_global_v2(xf + static_cast<size_t>(row + 8) * xrs + cc,
                                             v[16 * lh + 4 * j + 2], v[16 * lh + 4 * j + 3]);
                        }
                    }
                }
            }
            if (tid == 384) LA2_TR(17, s);
            return true;
        };

        if (Q::kOwnD) {
            // separate accumulators, no scaling in TMEM: X of tile s-1 is
            // written out (which frees X_inter for the next A W), then the state
            // update of tile s
            bool ok = true;
            for (int s = 0; s < ns && ok; ++s) {
                if (s > 0) ok = output(s - 1);
                ok = ok && update(s);
            }
            if (ok && ns > 0) output(ns - 1);
        } else {
            // dW sits in the X buffer of tile s+1, which tile s-1's X must leave first
            for (int s = 0; s < ns; ++s)
                if (!scale(s) || !update(s) || !output(s)) break;
        }
    }

    // ---- end of the segment: wait (bounded) until the issuers' MMAs are done
    __syncthreads();
    if (tid == 32 && ns > 0) {
        if (!mbar_wait(bar(Q::FIN), 0)) {
            *abort_flag = 1;
            atomicCAS(p.status, 0, 5 | (60 << 8));
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (*abort_flag) break;
    }  // segments

    // ---- tear-down: free TMEM
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (tid == 0) LA2_TR(18, 0);
}


// ---------------------------------------------------------------------------
// State pre-pass for segmented sequences.  One CTA per segment that ends
// inside its (sequence, role) unit.  The state a segment of n tiles leaves
// behind when it starts from zero is
//
//   S = sum_{s < n} lambda^(T_B (n-1-s)) (diag(w_s) B_s)^T C_s,
//
// so each tile's factor lambda^(T_B (n-1-s)) is folded into its row weights
// and all tiles accumulate into one TMEM accumulator: no per-tile state
// update, and B, lo(w B) and C are double-buffered.  S (fp32) goes to
// seg_state.  Roles (12 warps): warp 0 TMA (B, C), warp 1 MMA, warps 4-11 the
// weighted hi/lo split of B (two warps per TMEM lane quadrant, one per half
// of a row's 16-byte chunks), then the write-out of S.
constexpr int kStateThreads = 384;

enum StateBar { SB_B0, SB_B1, SB_C0, SB_C1, SB_S0, SB_S1, SB_D0, SB_D1, SB_FIN, SB_N };

template <int DA, int DC>
struct StateSmem {
    static constexpr uint32_t kBsz = kTB * DA * 2;
    static constexpr uint32_t kCsz = kTB * DC * 2;
    static constexpr uint32_t kB = 0;                     // B tiles (two), then hi(w B)
    static constexpr uint32_t kBlo = kB + 2 * kBsz;       // lo(w B) (two)
    static constexpr uint32_t kC = kBlo + 2 * kBsz;       // C tiles (two)
    static constexpr uint32_t kBar = kC + 2 * kCsz;
    static constexpr uint32_t kTmemSlot = kBar + SB_N * 8;
    static constexpr uint32_t kAbort = kTmemSlot + 4;
    static constexpr uint32_t kBytes = kAbort + 12;
    static constexpr uint32_t kTmemCols = DC;             // the S accumulator
};

template <int DA, int DC>
__global__ void __launch_bounds__(kStateThreads, 1)
la2_state_ws(const __grid_constant__ Params p)
{
    using L = StateSmem<DA, DC>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    if (base & 1023u) {
        if (threadIdx.x == 0) atomicCAS(p.status, 0, 4);
        return;
    }
    const uint32_t sB = base + L::kB, sBlo = base + L::kBlo, sC = base + L::kC;
    auto bar = [&](int b) { return base + L::kBar + 8u * b; };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem_raw + L::kAbort);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nb = (p.T + kTB - 1) / kTB;
    int unit, s0, ns;  // (sequence, role) and the segment's steps [s0, s0 + ns)
    long long slot;    // its slot in seg_state
    if (!p.balanced) {
        const int sj = blockIdx.x % (p.nseg - 1);
        unit = blockIdx.x / (p.nseg - 1);
        s0 = seg_begin(p, false, unit, sj, nb);
        ns = max(0, seg_begin(p, false, unit, sj + 1, nb) - s0);
        slot = seg_slot_index(p, false, unit, sj, nb);
    } else {
        // the segment that ends at boundary blockIdx.x + 1 of the scan's CTAs,
        // if that boundary falls inside a unit
        const long long gend = (static_cast<long long>(blockIdx.x) + 1) * p.seg_tiles;
        if (gend >= static_cast<long long>(p.nunits) * nb) return;
        unit = static_cast<int>(gend / nb);
        const int eloc = static_cast<int>(gend - static_cast<long long>(unit) * nb);
        if (eloc == 0) return;
        s0 = static_cast<int>(max(gend - p.seg_tiles, static_cast<long long>(unit) * nb) -
                              static_cast<long long>(unit) * nb);
        ns = eloc - s0;
        slot = blockIdx.x;
    }
    const int role_id = unit % p.nroles;
    const int bh = unit / p.nroles;
    const Role& R = p.role[role_id];
    const int dir = R.dir;
    const double l2 = log2(static_cast<double>(p.decay[bh % p.H]));
    auto tile_of = [&](int step) { return dir > 0 ? s0 + step : nb - 1 - (s0 + step); };

    if (warp == 0) {
        tmem_alloc(base + L::kTmemSlot, L::kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        const uint32_t counts[SB_N] = {1, 1, 1, 1, 256, 256, 1, 1, 1};
        for (int b = 0; b < SB_N; ++b) mbar_init(bar(b), counts[b]);
        *abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tD = *reinterpret_cast<volatile uint32_t*>(smem_raw + L::kTmemSlot);

    if (warp == 0) {
        // ================================================= TMA producer
        if (lane == 0 && ns > 0) {
            prefetch_tmap(&R.tb);
            prefetch_tmap(&R.tc);
            auto load = [&](int i, int slot) {
                const uint32_t bb = bar(SB_B0 + slot), bc = bar(SB_C0 + slot);
                mbar_arrive_expect_tx(bb, kTB * DA * 2);
                for (int gg = 0; gg < DA / 64; ++gg)
                    load_box(sB + slot * L::kBsz + gg * 16384, &R.tb, bb, gg * 64, i * kTB, bh, p.H, p.bthd);
                mbar_arrive_expect_tx(bc, kTB * DC * 2);
                for (int gg = 0; gg < DC / 64; ++gg)
                    load_box(sC + slot * L::kCsz + gg * 16384, &R.tc, bc, gg * 64, i * kTB, bh, p.H, p.bthd);
            };
            load(tile_of(0), 0);
            if (ns > 1) load(tile_of(1), 1);
            for (int s = 0; s + 2 < ns; ++s) {
                // buffers s % 2 are free once the MMAs of tile s are done
                if (!wait_bar(bar(SB_D0 + (s & 1)), (s >> 1) & 1, abort_flag, p.status, 70)) break;
                load(tile_of(s + 2), s & 1);
            }
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdW = idesc_bf16_f32(DA, DC, 1, 1);
            for (int s = 0; s < ns; ++s) {
                const int slot = s & 1;
                const uint32_t ph = (s >> 1) & 1;
                if (!wait_bar(bar(SB_S0 + slot), ph, abort_flag, p.status, 71)) break;
                if (!wait_bar(bar(SB_C0 + slot), ph, abort_flag, p.status, 72)) break;
                tc_fence_after();
                const uint32_t bh_ = sB + slot * L::kBsz, bl = sBlo + slot * L::kBsz;
                const uint32_t cb = sC + slot * L::kCsz;
#pragma unroll 1
                for (int k = 0; k < kTB / 16; ++k) {
                    const uint64_t cdesc = sdesc_sw128(cb + k * 2048, 16384, 1024);
                    mma_bf16_ss(tD, sdesc_sw128(bh_ + k * 2048, 16384, 1024), cdesc, kIdW,
                                (s > 0 || k > 0) ? 1u : 0u);
                    mma_bf16_ss(tD, sdesc_sw128(bl + k * 2048, 16384, 1024), cdesc, kIdW, 1);
                }
                mma_commit(bar(SB_D0 + slot));
            }
            mma_commit(bar(SB_FIN));
        }
    } else if (warp >= 4) {
        // ================================================= split group, then write-out
        const int quad = warp & 3, part = (warp - 4) >> 2;
        const int r = quad * 32 + lane;
        for (int s = 0; s < ns; ++s) {
            const int slot = s & 1;
            const uint32_t ph = (s >> 1) & 1;
            if (!wait_bar(bar(SB_B0 + slot), ph, abort_flag, p.status, 73)) break;
            // lo(w B) buffer of this slot was read by the MMAs of tile s-2
            if (s >= 2 && !wait_bar(bar(SB_D0 + slot), ph ^ 1, abort_flag, p.status, 74)) break;
            // row weight lambda^(T_B (n-1-s)) w_s(r)
            const int e = dir > 0 ? kTB * (ns - s) - 1 - r : kTB * (ns - 1 - s) + r;
            float wt = static_cast<float>(exp2(static_cast<double>(e) * l2));
            if (R.colf) {
                const int t = tile_of(s) * kTB + r;
                wt = t < p.T ? wt * __ldg(R.colf + static_cast<size_t>(bh) * p.T + t) : 0.f;
            }
            const uint32_t bt = sB + slot * L::kBsz, bl = sBlo + slot * L::kBsz;
#pragma unroll
            for (int k = 0; k < DA / 16; ++k) {
                const int chunk = part * (DA / 16) + k;
                const uint32_t off = (chunk >> 3) * 16384 + sw128(r, chunk & 7);
                uint32_t v[4], h[4], lo[4];
                ld_shared_v4(bt + off, v[0], v[1], v[2], v[3]);
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    split_pack2(bf16lo_to_f32(v[u]) * wt, bf16hi_to_f32(v[u]) * wt, h[u], lo[u]);
                st_shared_v4(bt + off, h[0], h[1], h[2], h[3]);
                st_shared_v4(bl + off, lo[0], lo[1], lo[2], lo[3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(bar(SB_S0 + slot));
        }
        // S of this segment: TMEM -> seg_state (fp32, row-major DA x DC)
        if (ns > 0 &&
            wait_bar(bar(SB_D0 + ((ns - 1) & 1)), ((ns - 1) >> 1) & 1, abort_flag, p.status, 75)) {
            tc_fence_after();
            const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
            const bool owns_row = (DA == 128) || (lane < 16);
            const int srow = (DA == 128) ? r : quad * 16 + (lane & 15);
            float* dst0 = p.seg_state + static_cast<size_t>(slot) * (DA * DC) + static_cast<size_t>(srow) * DC;
#pragma unroll 1
            for (int k = 0; k < DC / 32; ++k) {
                const int col = part * (DC / 2) + k * 16;
                float w[16];
                tmem_ld16(tD + lane_off + col, w);
                if (owns_row) {
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        st_global_v4(dst0 + col + 4 * u, w[4 * u], w[4 * u + 1], w[4 * u + 2],
                                     w[4 * u + 3]);
                }
            }
        }
    }

    __syncthreads();
    if (tid == 32 && ns > 0) {
        if (!mbar_wait(bar(SB_FIN), 0)) atomicCAS(p.status, 0, 5 | (76 << 8));
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tD, L::kTmemCols);
    }
}

}  // namespace ws
}  // namespace la2
