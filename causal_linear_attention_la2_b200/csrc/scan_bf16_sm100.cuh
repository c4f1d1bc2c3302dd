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
// the decay-weighted factor of the state update) are fp32 values; each is fed to the tensor core as the sum of
// two bf16 terms (hi + lo, relative residue ~2^-16), i.e. as two MMAs.
//
// Work split: one CTA per (sequence, role, 64-column slice of c/x).  Each CTA
// runs its tiles serially (the state makes the scan sequential); two CTAs fit
// on an SM (256 TMEM columns, <= 113 KB of shared memory and 256 threads of
// <= 128 registers each), so one CTA's TMA traffic overlaps the other's math.
// Two threads share each tile row (TMEM lane), one per half of its columns.
//
// Shared-memory tiles are 128-byte swizzled, as TMA writes them; the A and B
// tiles serve both K-major (for S) and MN-major (for the state update)
// descriptors.  Once S and A W are computed the A buffer takes the hi and lo
// parts of the weighted factor of the state update; the C buffer stages the
// fp32 X tile for its TMA stores once the MMAs are done with it.  P (hi and lo) lives in TMEM over the columns
// of S it was computed from and feeds the MMA as its A operand from TMEM.
#pragma once
#include "ptx_sm100.cuh"

namespace la2 {

constexpr int kTB = 128;        // tile length T_B of this kernel
constexpr int kSlice = 64;      // columns of c / x per CTA
constexpr int kThreads = 256;   // two threads per TMEM lane / tile row
constexpr uint32_t kTmemCols = 256;

struct ScanRole {
    CUtensorMap ta, tb, tc;  // a, b: [B*H, T, DA]; c: [B*H, T, DC]; bf16, box 64 x 128
    CUtensorMap tx;          // x: [B*H, T, DC] fp32, box 32 x 128
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

// The state update needs diag(w_s) B_i^T C_i with one of the two factors
// weighted and split into hi + lo.  With DA = 128 the C slice (64 columns) is
// the smaller one and its hi/lo pair fits the A buffer; with DA = 64 the B
// tile is split (hi in place, lo in the A buffer).
template <int DA>
struct ScanSmem {
    static constexpr bool kSplitC = (DA == 128);
    static constexpr uint32_t kA = 0;          // A tile, then the hi/lo split, then X staging
    static constexpr uint32_t kB = kA + 32768;                // B tile
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
__global__ void __launch_bounds__(kThreads, 2)
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
    const int quad = warp & 3;   // TMEM lane quadrant this warp may access
    const int half = warp >> 2;  // which half of a row's columns this thread handles
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
        mbar_init(bar_mma, 2);  // both MMA-issuing threads commit to it
        fence_mbar_init();
        prefetch_tmap(&R.ta);
        prefetch_tmap(&R.tb);
        prefetch_tmap(&R.tc);
        prefetch_tmap(&R.tx);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tX = tmem + 128, tD = tmem + 192;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const float lamTB = pw[kTB];

    constexpr uint32_t kTxBytes = 2u * kTB * DA * 2 + kTB * kSlice * 2;
    constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, 0, 0);    // S  = A B^T
    constexpr uint32_t kIdX = idesc_bf16_f32(128, kSlice, 0, 1);  // X += P C
    constexpr uint32_t kIdXW = idesc_bf16_f32(128, 2 * kSlice, 0, 1);  // [X | X'] = A [hi(W) | lo(W)]
    constexpr uint32_t kIdW = idesc_bf16_f32(DA, kSlice, 1, 1);   // dW = B^T C

    // One phase of bar_load covers A, B and C of a tile; C may be issued later
    // than A and B (its buffer stages the previous tile's X store).
    auto issue_loads_ab = [&](int i) {
        mbar_arrive_expect_tx(bar_load, kTxBytes);
#pragma unroll
        for (int g = 0; g < DA / 64; ++g) {
            tma_load_3d(sA + g * 16384, &R.ta, bar_load, g * 64, i * kTB, bh);
            tma_load_3d(sB + g * 16384, &R.tb, bar_load, g * 64, i * kTB, bh);
        }
    };
    auto issue_loads_c = [&](int i) { tma_load_3d(sC, &R.tc, bar_load, x0, i * kTB, bh); };

    if (tid == 0 && nb > 0) {
        issue_loads_ab(dir > 0 ? 0 : nb - 1);
        issue_loads_c(dir > 0 ? 0 : nb - 1);
    }

    float w[32];  // fp32 state: row wrow of W, columns [32*half, 32*half + 32) of this slice
#pragma unroll
    for (int c = 0; c < 32; ++c) w[c] = 0.f;
    const bool owns_w_row = (DA == 128) || (lane < 16);
    const int wrow = (DA == 128) ? quad * 32 + lane : quad * 16 + (lane & 15);

    const int r = quad * 32 + lane;  // tile row handled by this thread
    // Two threads issue tcgen05.mma, each its own accumulator chain: one
    // issuing thread sustains ~1 MMA per 100 cycles at these shapes, two
    // overlap.  Issuer 0 is thread 0 (warp 0), issuer 1 thread 128 (warp 4).
    const bool issuer0 = tid == 0, issuer1 = tid == 128;
    uint32_t ph_load = 0, ph_mma = 0;

    for (int step = 0; step < nb; ++step) {
        const int i = dir > 0 ? step : nb - 1 - step;

        // (1) tiles A_i, B_i, C_i have landed
        bool ok = true;
        if (tid == 0) ok = mbar_wait(bar_load, ph_load);
        ph_load ^= 1;
        if (!__syncthreads_and(ok)) {
            if (tid == 0) report_status(p.status, kDevTimeout, 1);
            break;
        }

        // (2) issuer 0: S = A B^T.  issuer 1: [X | X'] = A [hi(W) | lo(W)], one
        //     N = 128 MMA per K step whose two halves land in the X columns and
        //     in the (still free) dW columns next to them.
        if (issuer0 || issuer1) {
            tc_fence_after();
#pragma unroll 1
            for (int s = 0; s < DA / 16; ++s) {
                const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                const uint64_t adesc = sdesc_sw128(sA + off, 16, 1024);
                if (issuer0)
                    mma_bf16_ss(tS, adesc, sdesc_sw128(sB + off, 16, 1024), kIdS, s > 0);
                else
                    mma_bf16_ss(tX, adesc, sdesc_sw128(sWhi + s * 2048, DA * kSlice * 2, 1024),
                                kIdXW, s > 0);
            }
            mma_commit(bar_mma);
        }
        if (tid == 0) ok = mbar_wait(bar_mma, ph_mma);
        ph_mma ^= 1;
        if (!__syncthreads_and(ok)) {
            if (tid == 0) report_status(p.status, kDevTimeout, 2);
            break;
        }
        tc_fence_after();

        // (3a) P = decay-masked S as hi + lo bf16, written into TMEM over the
        //     16 columns of S each group of 16 came from: [hi (8 cols) | lo (8 cols)],
        //     which is the A-operand layout of one K=16 step.  This thread does
        //     groups 4*half .. 4*half+3 of row r.  Every group is loaded before it
        //     is overwritten, also groups the mask zeroes entirely: storing over S
        //     columns that were not read first made the following TMEM-operand
        //     MMAs about 10x slower.
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int g = 4 * half + k;
            // warp-uniform group kind: 0 = all masked, 1 = crosses the diagonal, 2 = all causal
            const int lo_g = 2 * quad, hi_g = 2 * quad + 1;
            const int kind = (g == lo_g || g == hi_g) ? 1 : ((dir > 0) == (g < lo_g) ? 2 : 0);
            uint32_t pk[16];
            float s[16];
            tmem_ld16(tS + lane_off + g * 16, s);
            if (kind == 2) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int c0 = g * 16 + 2 * u;
                    const float p0 = s[2 * u] * pw[dir > 0 ? r - c0 : c0 - r];
                    const float p1 = s[2 * u + 1] * pw[dir > 0 ? r - c0 - 1 : c0 + 1 - r];
                    split_pack2(p0, p1, pk[u], pk[8 + u]);
                }
            } else if (kind == 1) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int c0 = g * 16 + 2 * u;
                    const int lag0 = dir > 0 ? r - c0 : c0 - r;
                    const int lag1 = dir > 0 ? r - c0 - 1 : c0 + 1 - r;
                    const float p0 = lag0 >= 0 ? s[2 * u] * pw[lag0 < 0 ? 0 : lag0] : 0.f;
                    const float p1 = lag1 >= 0 ? s[2 * u + 1] * pw[lag1 < 0 ? 0 : lag1] : 0.f;
                    split_pack2(p0, p1, pk[u], pk[8 + u]);
                }
            } else {
#pragma unroll
                for (int u = 0; u < 16; ++u) pk[u] = 0u;
            }
            tmem_st16(tS + lane_off + g * 16, pk);
        }

        // (3b) X row r = w_x(r) (X + X')   (the inter-tile term, still alone in X)
        {
            const float wx = dir > 0 ? pw[r + 1] : pw[kTB - r];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                float x[16], y[16];
                const uint32_t col = half * 32 + k * 16;
                tmem_ld16(tX + lane_off + col, x);
                tmem_ld16(tD + lane_off + col, y);
#pragma unroll
                for (int u = 0; u < 16; ++u) x[u] = (x[u] + y[u]) * wx;
                tmem_st16f(tX + lane_off + col, x);
            }
        }

        // (3c) row r of the weighted factor of the state update, split hi/lo;
        //      this thread does 16-byte chunks 4*half .. 4*half+3 of the row
        {
            const float ws = dir > 0 ? pw[kTB - 1 - r] : pw[r];
            const uint32_t src = L::kSplitC ? sC : sB;
            const uint32_t dst_hi = L::kSplitC ? sA : sB;
            const uint32_t dst_lo = L::kSplitC ? sA + 16384 : sA;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t off = sw128(r, 4 * half + k);
                uint32_t v[4], h[4], l[4];
                ld_shared_v4(src + off, v[0], v[1], v[2], v[3]);
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    split_pack2(bf16lo_to_f32(v[u]) * ws, bf16hi_to_f32(v[u]) * ws, h[u], l[u]);
                st_shared_v4(dst_hi + off, h[0], h[1], h[2], h[3]);
                st_shared_v4(dst_lo + off, l[0], l[1], l[2], l[3]);
            }
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // (4) issuer 0: X += hi(P) C + lo(P) C.  issuer 1: dW = B^T hi(w_s C) +
        //     B^T lo(w_s C)  (DA = 64: dW = hi(w_s B)^T C + lo(w_s B)^T C).
        if (issuer0 || issuer1) {
            tc_fence_after();
#pragma unroll 1
            for (int s = 0; s < kTB / 16; ++s) {
                const uint64_t cdesc = sdesc_sw128(sC + s * 2048, 16384, 1024);
                if (issuer0) {
                    const uint32_t pcol = s * 16;  // hi(P) at pcol, lo(P) at pcol + 8
                    mma_bf16_ts(tX, tS + pcol, cdesc, kIdX, 1);
                    mma_bf16_ts(tX, tS + pcol + 8, cdesc, kIdX, 1);
                } else if (L::kSplitC) {
                    const uint64_t bdesc = sdesc_sw128(sB + s * 2048, 16384, 1024);
                    mma_bf16_ss(tD, bdesc, sdesc_sw128(sA + s * 2048, 16384, 1024), kIdW, s > 0);
                    mma_bf16_ss(tD, bdesc, sdesc_sw128(sA + 16384 + s * 2048, 16384, 1024), kIdW, 1);
                } else {
                    mma_bf16_ss(tD, sdesc_sw128(sB + s * 2048, 16384, 1024), cdesc, kIdW, s > 0);
                    mma_bf16_ss(tD, sdesc_sw128(sA + s * 2048, 16384, 1024), cdesc, kIdW, 1);
                }
            }
            mma_commit(bar_mma);
        }
        if (tid == 0) ok = mbar_wait(bar_mma, ph_mma);
        ph_mma ^= 1;
        if (!__syncthreads_and(ok)) {
            if (tid == 0) report_status(p.status, kDevTimeout, 3);
            break;
        }
        tc_fence_after();

        // (5) A and B buffers are free: start the next tile's A, B loads (C
        //     follows once the X staging in the C buffer has been read)
        const bool has_next = step + 1 < nb;
        const int inext = dir > 0 ? i + 1 : i - 1;
        if (tid == 0 && has_next) issue_loads_ab(inext);

        // (6a) X leaves through the C buffer, one 128 x 32 fp32 box (16 KB,
        //      128-byte swizzled) per round: in round k the threads of half k
        //      write their 32 columns, thread 0 issues the TMA store (rows past
        //      T are clipped) and waits until the box has been read.
        {
            float x[32];
            tmem_ld32(tX + lane_off + half * 32, x);
#pragma unroll 1
            for (int k = 0; k < 2; ++k) {
                if (half == k) {
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        st_shared_v4(sC + sw128(r, q), __float_as_uint(x[4 * q]),
                                     __float_as_uint(x[4 * q + 1]), __float_as_uint(x[4 * q + 2]),
                                     __float_as_uint(x[4 * q + 3]));
                    fence_proxy_async_smem();
                }
                __syncthreads();
                if (tid == 0) {
                    tma_store_3d(&R.tx, sC, x0 + 32 * k, i * kTB, bh);
                    bulk_commit();
                    bulk_wait_read0();
                }
                __syncthreads();
            }
        }
        if (tid == 0 && has_next) issue_loads_c(inext);

        // (6b) W <- lambda^T_B W + dW (fp32, registers); hi/lo bf16 copies for the next tile
        {
            float dw[32];
            tmem_ld32(tD + lane_off + half * 32, dw);
#pragma unroll
            for (int u = 0; u < 32; ++u) w[u] = fmaf(lamTB, w[u], dw[u]);
            if (owns_w_row) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint32_t h[4], l[4];
#pragma unroll
                    for (int z = 0; z < 4; ++z)
                        split_pack2(w[8 * u + 2 * z], w[8 * u + 2 * z + 1], h[z], l[z]);
                    const uint32_t off = sw128(wrow, 4 * half + u);
                    st_shared_v4(sWhi + off, h[0], h[1], h[2], h[3]);
                    st_shared_v4(sWlo + off, l[0], l[1], l[2], l[3]);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    if (tid == 0) bulk_wait0();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace la2
