// scan_bf16_sm100.cuh -- the bf16-input tcgen05 kernel of the Lightning
// Attention-2 hot path.
//
// One kernel computes every output of the forward and the backward pass as a
// "decayed scan" over tiles of T_B = 128 rows:
//
//   dir = +1:  x_t = sum_{s<=t} lambda^(t-s) (a_t . b_s) c_s
//   dir = -1:  x_t = sum_{s>=t} lambda^(s-t) (a_t . b_s) c_s
//
//   forward  o  = scan(+1; a=q,  b=k,  c=v)
//   backward dq = scan(+1; a=dO, b=v,  c=k)
//            dk = scan(-1; a=v,  b=dO, c=q)
//            dv = scan(-1; a=k,  b=q,  c=dO)
//
// Per tile i (rows r, columns c local to the tile), following the tiled
// derivation of the "Lightning Attention" page (lizeman.github.io llm-arch-kb,
// section 2, steps 1-4) with the decay folded in:
//
//   S   = A_i B_i^T                                   tcgen05, fp32 in TMEM
//   P   = S * lambda^|r-c| on the causal side, else 0 registers -> TMEM
//   X   = diag(w_x) A_i W + P C_i                     tcgen05, fp32 in TMEM
//   W  <- lambda^T_B W + (diag(w_s) B_i)^T C_i        tcgen05 + fp32 registers
//
// with w_x = lambda^(r+1), w_s = lambda^(T_B-1-r) for dir = +1 and
// w_x = lambda^(T_B-r), w_s = lambda^r for dir = -1.  W is the d x e state,
// carried on chip in fp32 for the whole sequence; nothing per tile goes back
// to HBM except X, which is written in fp32.
//
// Precision: inputs are bf16 and every product of two inputs is exact in the
// fp32 accumulators.  The three operands the kernel forms itself (P, W and
// diag(w_s) B) are fp32 values; each is fed to the tensor core as the sum of
// two bf16 terms (hi + lo, relative residue ~2^-16), i.e. as two MMAs.
//
// Work split: one CTA per (sequence, role, 64-column slice of c/x).  Each CTA
// runs its tiles serially (the state makes the scan sequential); two CTAs fit
// on an SM (256 TMEM columns and ~113 KB of shared memory each), so one CTA's
// TMA traffic overlaps the other's math.
//
// Shared-memory tiles are 128-byte swizzled, as TMA writes them; the A and B
// tiles serve both K-major (for S) and MN-major (for the state update)
// descriptors.  Once S and A W are computed the A buffer takes the lo part of
// diag(w_s) B, and the B buffer its hi part in place.  P (hi and lo) lives in
// TMEM over the columns of S it was computed from and feeds the MMA as its A
// operand straight from TMEM.
#pragma once
#include "ptx_sm100.cuh"

namespace la2 {

constexpr int kTB = 128;        // tile length T_B of this kernel
constexpr int kSlice = 64;      // columns of c / x per CTA
constexpr int kThreads = 128;   // one thread per TMEM lane / tile row
constexpr uint32_t kTmemCols = 256;

struct ScanRole {
    CUtensorMap ta, tb, tc;  // a, b: [B*H, T, DA]; c: [B*H, T, DC]; bf16
    float* x;                // [B*H, T, DC] fp32
    int dir;                 // +1 or -1
};

struct ScanParams {
    ScanRole role[3];
    const float* decay;  // [H]
    int* status;         // device status word
    int H, T, nroles, nslices, dc;
};

// Device status codes: low byte = la2_status, next byte = where.
constexpr int kDevTimeout = 5;
constexpr int kDevMisaligned = 4;
__device__ __forceinline__ void report_status(int* status, int code, int where) {
    atomicCAS(status, 0, code | (where << 8));
}

// Byte offset of the 16-byte chunk q (0..7) of row r inside a 128-byte
// swizzled region (rows of 128 bytes, 8-row groups of 1024 bytes).
__device__ __forceinline__ uint32_t sw128(int r, int q) {
    return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((q ^ (r & 7)) << 4));
}

template <int DA>
struct ScanSmem {
    static constexpr uint32_t kA = 0;                         // A tile, then lo(w_s B)
    static constexpr uint32_t kB = kA + kTB * DA * 2;         // B tile, then hi(w_s B)
    static constexpr uint32_t kC = kB + kTB * DA * 2;         // C slice (T_B x 64)
    static constexpr uint32_t kWhi = kC + kTB * kSlice * 2;   // hi(W) (DA x 64)
    static constexpr uint32_t kWlo = kWhi + DA * kSlice * 2;  // lo(W)
    static constexpr uint32_t kPow = kWlo + DA * kSlice * 2;  // lambda^n, n = 0..T_B
    static constexpr uint32_t kBarLoad = kPow + 528;
    static constexpr uint32_t kBarMma = kBarLoad + 8;
    static constexpr uint32_t kTmemSlot = kBarMma + 8;
    static constexpr uint32_t kEnd = kTmemSlot + 16;
    // The dynamic shared memory base is 1024-byte aligned (checked at run
    // time).  Small tiles are padded so that at most two CTAs share an SM:
    // their TMEM then adds up to the SM's 512 columns.
    static constexpr uint32_t kBytes = kEnd > 78 * 1024 ? kEnd : 78 * 1024;
};

template <int DA>
__global__ void __launch_bounds__(kThreads, 1)
la2_scan_bf16_sm100(const __grid_constant__ ScanParams p)
{
    static_assert(DA == 64 || DA == 128, "DA must be 64 or 128");
    using L = ScanSmem<DA>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    if (base & 1023u) {  // 128-byte swizzled tiles need a 1024-byte aligned base
        if (threadIdx.x == 0) report_status(p.status, kDevMisaligned, 0);
        return;
    }

    const uint32_t sA = base + L::kA, sB = base + L::kB, sC = base + L::kC;
    const uint32_t sWhi = base + L::kWhi, sWlo = base + L::kWlo;
    float* pw = reinterpret_cast<float*>(smem_raw + L::kPow);
    const uint32_t bar_load = base + L::kBarLoad, bar_mma = base + L::kBarMma;
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem_raw + L::kTmemSlot);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int idx = blockIdx.x;
    const int slice = idx % p.nslices;
    idx /= p.nslices;
    const int role = idx % p.nroles;
    const int bh = idx / p.nroles;
    const ScanRole& R = p.role[role];
    const int dir = R.dir;
    const int T = p.T;
    const int nb = (T + kTB - 1) / kTB;
    const int x0 = slice * kSlice;
    const float lam = p.decay[bh % p.H];
    float* xg = R.x + static_cast<size_t>(bh) * T * p.dc + x0;

    // ---- set-up: powers of lambda, zero state copy, barriers, TMEM
    {
        const double l2 = log2(static_cast<double>(lam));
        for (int n = tid; n <= kTB; n += kThreads) pw[n] = static_cast<float>(exp2(n * l2));
        for (uint32_t off = tid * 16; off < static_cast<uint32_t>(2 * DA * kSlice * 2);
             off += kThreads * 16)
            st_shared_v4(sWhi + off, 0u, 0u, 0u, 0u);  // hi(W) and lo(W) are adjacent
    }
    if (warp == 0) {
        tmem_alloc(base + L::kTmemSlot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_load, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        prefetch_tmap(&R.ta);
        prefetch_tmap(&R.tb);
        prefetch_tmap(&R.tc);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tX = tmem + 128, tD = tmem + 192;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float lamTB = pw[kTB];

    constexpr uint32_t kTxBytes = 2u * kTB * DA * 2 + kTB * kSlice * 2;
    constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, 0, 0);    // S  = A B^T
    constexpr uint32_t kIdX = idesc_bf16_f32(128, kSlice, 0, 1);  // X  = A W, X += P C
    constexpr uint32_t kIdW = idesc_bf16_f32(DA, kSlice, 1, 1);   // dW = B^T C

    auto issue_loads = [&](int i) {
        mbar_arrive_expect_tx(bar_load, kTxBytes);
#pragma unroll
        for (int g = 0; g < DA / 64; ++g) {
            tma_load_3d(sA + g * 16384, &R.ta, bar_load, g * 64, i * kTB, bh);
            tma_load_3d(sB + g * 16384, &R.tb, bar_load, g * 64, i * kTB, bh);
        }
        tma_load_3d(sC, &R.tc, bar_load, x0, i * kTB, bh);
    };

    if (tid == 0 && nb > 0) issue_loads(dir > 0 ? 0 : nb - 1);

    float w[kSlice];  // fp32 state row (row j of W, this CTA's 64 columns)
#pragma unroll
    for (int c = 0; c < kSlice; ++c) w[c] = 0.f;
    const bool owns_w_row = (DA == 128) || (lane < 16);
    const int wrow = (DA == 128) ? tid : warp * 16 + (lane & 15);

    const int r = tid;  // tile row handled by this thread
    uint32_t ph_load = 0, ph_mma = 0;

    for (int step = 0; step < nb; ++step) {
        const int i = dir > 0 ? step : nb - 1 - step;
        const int rows = min(kTB, T - i * kTB);

        // (1) tiles A_i, B_i, C_i have landed
        bool ok = true;
        if (tid == 0) ok = mbar_wait(bar_load, ph_load);
        ph_load ^= 1;
        if (!__syncthreads_and(ok)) {
            if (tid == 0) report_status(p.status, kDevTimeout, 1);
            break;
        }

        // (2) S = A B^T;  X = A hi(W) + A lo(W)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < DA / 16; ++s) {
                const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                mma_bf16_ss(tS, sdesc_sw128(sA + off, 16, 1024), sdesc_sw128(sB + off, 16, 1024),
                            kIdS, s > 0);
            }
#pragma unroll
            for (int s = 0; s < DA / 16; ++s) {
                const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                mma_bf16_ss(tX, sdesc_sw128(sA + off, 16, 1024),
                            sdesc_sw128(sWhi + s * 2048, 16384, 1024), kIdX, s > 0);
            }
#pragma unroll
            for (int s = 0; s < DA / 16; ++s) {
                const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                mma_bf16_ss(tX, sdesc_sw128(sA + off, 16, 1024),
                            sdesc_sw128(sWlo + s * 2048, 16384, 1024), kIdX, 1);
            }
            mma_commit(bar_mma);
            ok = mbar_wait(bar_mma, ph_mma);
        }
        ph_mma ^= 1;
        if (!__syncthreads_and(ok)) {
            if (tid == 0) report_status(p.status, kDevTimeout, 2);
            break;
        }
        tc_fence_after();

        // (3a) P = decay-masked S as hi + lo bf16, written into TMEM over the
        //      32 columns of S each chunk came from: [hi (16 cols) | lo (16 cols)]
        //      Every chunk is loaded before it is overwritten, also chunks the
        //      mask zeroes entirely: storing over S columns that were not read
        //      first made the following TMEM-operand MMAs about 10x slower.
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            uint32_t hi[16], lo[16];
            float s[32];
            tmem_ld32(tS + lane_off + cc * 32, s);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int c0 = cc * 32 + 2 * u;
                const int lag0 = dir > 0 ? r - c0 : c0 - r;
                const int lag1 = dir > 0 ? r - c0 - 1 : c0 + 1 - r;
                const float p0 = lag0 >= 0 ? s[2 * u] * pw[lag0 < 0 ? 0 : lag0] : 0.f;
                const float p1 = lag1 >= 0 ? s[2 * u + 1] * pw[lag1 < 0 ? 0 : lag1] : 0.f;
                split_pack2(p0, p1, hi[u], lo[u]);
            }
            tmem_st16(tS + lane_off + cc * 32, hi);
            tmem_st16(tS + lane_off + cc * 32 + 16, lo);
        }

        // (3b) X row r *= w_x(r)   (the inter-tile term, still alone in X)
        {
            const float wx = dir > 0 ? pw[r + 1] : pw[kTB - r];
#pragma unroll
            for (int cc = 0; cc < kSlice / 32; ++cc) {
                float x[32];
                tmem_ld32(tX + lane_off + cc * 32, x);
#pragma unroll
                for (int u = 0; u < 32; ++u) x[u] *= wx;
                tmem_st32(tX + lane_off + cc * 32, x);
            }
        }

        // (3c) row r of w_s(r) B: hi part in place in the B buffer, lo part
        //      into the (now free) A buffer at the same offset
        {
            const float ws = dir > 0 ? pw[kTB - 1 - r] : pw[r];
#pragma unroll
            for (int g = 0; g < DA / 64; ++g) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint32_t off = g * 16384 + sw128(r, q);
                    uint32_t v[4], h[4], l[4];
                    ld_shared_v4(sB + off, v[0], v[1], v[2], v[3]);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        split_pack2(bf16lo_to_f32(v[u]) * ws, bf16hi_to_f32(v[u]) * ws, h[u], l[u]);
                    st_shared_v4(sB + off, h[0], h[1], h[2], h[3]);
                    st_shared_v4(sA + off, l[0], l[1], l[2], l[3]);
                }
            }
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // (4) X += hi(P) C + lo(P) C;  dW = hi(w_s B)^T C + lo(w_s B)^T C
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < kTB / 16; ++s) {
                const uint32_t pcol = (s >> 1) * 32 + (s & 1) * 8;
                const uint64_t cdesc = sdesc_sw128(sC + s * 2048, 16384, 1024);
                mma_bf16_ts(tX, tS + pcol, cdesc, kIdX, 1);
                mma_bf16_ts(tX, tS + pcol + 16, cdesc, kIdX, 1);
            }
#pragma unroll
            for (int s = 0; s < kTB / 16; ++s) {
                const uint64_t cdesc = sdesc_sw128(sC + s * 2048, 16384, 1024);
                mma_bf16_ss(tD, sdesc_sw128(sB + s * 2048, 16384, 1024), cdesc, kIdW, s > 0);
                mma_bf16_ss(tD, sdesc_sw128(sA + s * 2048, 16384, 1024), cdesc, kIdW, 1);
            }
            mma_commit(bar_mma);
            ok = mbar_wait(bar_mma, ph_mma);
        }
        ph_mma ^= 1;
        if (!__syncthreads_and(ok)) {
            if (tid == 0) report_status(p.status, kDevTimeout, 3);
            break;
        }
        tc_fence_after();

        // (5) all smem tiles are free: start the next tile's loads
        if (tid == 0 && step + 1 < nb) issue_loads(dir > 0 ? i + 1 : i - 1);

        // (6a) X row r -> fp32 -> global (rows past T are not stored)
#pragma unroll
        for (int cc = 0; cc < kSlice / 32; ++cc) {
            float x[32];
            tmem_ld32(tX + lane_off + cc * 32, x);
            if (r < rows) {
                float* dst = xg + static_cast<size_t>(i * kTB + r) * p.dc + cc * 32;
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    st_global_v4(dst + 4 * u, x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]);
            }
        }

        // (6b) W <- lambda^T_B W + dW (fp32, registers); hi/lo bf16 copies for the next tile
#pragma unroll
        for (int cc = 0; cc < kSlice / 32; ++cc) {
            float dw[32];
            tmem_ld32(tD + lane_off + cc * 32, dw);
#pragma unroll
            for (int u = 0; u < 32; ++u) w[cc * 32 + u] = fmaf(lamTB, w[cc * 32 + u], dw[u]);
            if (owns_w_row) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int c = cc * 32 + u * 8;
                    uint32_t h[4], l[4];
#pragma unroll
                    for (int z = 0; z < 4; ++z)
                        split_pack2(w[c + 2 * z], w[c + 2 * z + 1], h[z], l[z]);
                    const uint32_t off = sw128(wrow, cc * 4 + u);
                    st_shared_v4(sWhi + off, h[0], h[1], h[2], h[3]);
                    st_shared_v4(sWlo + off, l[0], l[1], l[2], l[3]);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace la2
