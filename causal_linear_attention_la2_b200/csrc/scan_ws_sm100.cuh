// scan_ws_sm100.cuh -- warp-specialised bf16-input tcgen05 kernel of the
// Lightning Attention-2 hot path: one CTA per SM and per (sequence, role),
// the whole value width (DC = 64 or 128) in one CTA, tiles of T_B = 128 rows.
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
//   P   = S * lambda^|r-c| on the causal side, else 0 (registers -> TMEM, hi + lo bf16)
//   X   = diag(w_x) A_i W + P C_i                   (tcgen05, TMEM, fp32)
//   dW  = (diag(w_s) B_i)^T C_i                     (tcgen05, TMEM; hi + lo of w_s B)
//   W  <- lambda^T_B W + dW                         (fp32 arithmetic; W kept as hi + lo bf16)
//
// with w_x = lambda^(r+1), w_s = lambda^(T_B-1-r) for dir = +1 and
// w_x = lambda^(T_B-r), w_s = lambda^r for dir = -1.
//
// Roles (20 warps):
//   warp 0      TMA producer: A and C (one buffer each), B (two buffers)
//   warp 3      MMA issuer 0: S (two TMEM buffers, so S of the next tile is
//               formed while P C of this one is still pending)
//   warp 1      MMA issuer 1: X += P C
//   warp 2      MMA issuer 2: X = A hi(W) + A lo(W) (X double-buffered in
//               TMEM), dW = hi(w_s B)^T C + lo(w_s B)^T C (into the X buffer
//               the next tile will use)
//   warps 4-11  mask group (two warps per TMEM lane quadrant): P from S, then
//               the hi/lo split of w_s B (hi in place, lo in its own buffer)
//   warps 12-19 epilogue group (two warps per lane quadrant, one per half of
//               the columns): X = w_x X, the W update (W lives in shared
//               memory as the hi/lo bf16 pair the next X MMA reads), X to global
//               memory in fp32 (a warp-shuffle transpose makes every store a
//               whole 128-byte row)
// Tile i's epilogue overlaps tile i+1's loads, S and P; each issuer waits only
// for the operands of its own MMAs, so no MMA queues behind an unrelated one.
//
// Every hand-off is an mbarrier; every wait is bounded (2 s) and a shared abort
// flag stops all roles once one of them gives up, after which the kernel
// waits (bounded) for its own MMAs, frees TMEM and returns.
#pragma once
#include "ptx_sm100.cuh"

namespace la2 {
namespace ws {

constexpr int kTB = 128;
constexpr int kThreads = 640;
constexpr uint32_t kTmemCols = 512;

struct Role {
    CUtensorMap ta, tb, tc;  // a, b: [B*H, T, DA]; c: [B*H, T, DC]; bf16, box 64 x 128
    float* x;                // [B*H, T, DC] fp32
    int dir;                 // +1 or -1
};

struct Params {
    Role role[3];
    const float* decay;  // [H]
    int* status;         // device status word
    float* seg_state;    // [B*H][nroles][nseg - 1][DA][DC] fp32: local end state of each
                         // segment but the last (written by the state pass)
    int H, T, nroles;
    int nseg;            // segments per (sequence, role); 1 = no split
    int seg_tiles;       // tiles per segment (the last may be shorter)
};

enum Bar {
    FULL_A, FULL_B0, FULL_B1, FULL_C,  // TMA loads landed
    B_S0, B_S1, B_X0, B_X1, B_PC0, B_PC1, B_D,  // MMA commits: S (per S buffer); X = A W (per
                                                // X buffer); X += P C (per S buffer); dW
    B_P0, B_P1, B_BS,                    // mask: P written (per S buffer), w_s B split
    B_XS, B_WR, B_XF0, B_XF1,          // epilogue: X scaled; W updated (dW read); X buffer 0 / 1 read
    B_FIN, NBAR
};

template <int DA, int DC>
struct Smem {
    static constexpr uint32_t kA = 0;                        // A tile (T_B x DA)
    static constexpr uint32_t kBsz = kTB * DA * 2;
    static constexpr uint32_t kB = kA + kBsz;                // B tiles, two buffers, each then hi(w_s B)
    static constexpr uint32_t kBlo = kB + 2 * kBsz;          // lo(w_s B)
    static constexpr uint32_t kC = kBlo + kBsz;              // C tile (T_B x DC)
    static constexpr uint32_t kWsz = DA * DC * 2;
    static constexpr uint32_t kW = kC + kTB * DC * 2;        // hi(W), then lo(W) (DA x DC each)
    static constexpr uint32_t kPow = kW + 2 * kWsz;          // lambda^n, n = 0..T_B
    static constexpr uint32_t kBar = kPow + 528;
    static constexpr uint32_t kTmemSlot = kBar + NBAR * 8;
    static constexpr uint32_t kAbort = kTmemSlot + 4;
    static constexpr uint32_t kEnd = kAbort + 12;
    // Small tiles are padded so that only one CTA fits on an SM (it allocates
    // all 512 TMEM columns).
    static constexpr uint32_t kBytes = kEnd > 120 * 1024 ? kEnd : 120 * 1024;
};

// Byte offset of the 16-byte chunk q (0..7) of row r inside a 128-byte
// swizzled region (rows of 128 bytes, 8-row groups of 1024 bytes).
__device__ __forceinline__ uint32_t sw128(int r, int q) {
    return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((q ^ (r & 7)) << 4));
}

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         int* status, int where) {
    if (mbar_try_wait_hint(bar, parity, 64)) return true;
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

// The scan itself.  One CTA per (sequence, role, segment); a segment starts
// from the state the segments before it leave behind,
// W_in(g) = sum_{g' < g} lambda^(T_B n (g-1-g')) S_g' (n tiles per segment),
// read from seg_state (written by la2_state_ws).
template <int DA, int DC>
__global__ void __launch_bounds__(kThreads, 1)
la2_scan_ws(const __grid_constant__ Params p)
{
    static_assert((DA == 64 || DA == 128) && (DC == 64 || DC == 128), "DA, DC in {64, 128}");
    using L = Smem<DA, DC>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    if (base & 1023u) {  // 128-byte swizzled tiles need a 1024-byte aligned base
        if (threadIdx.x == 0) atomicCAS(p.status, 0, 4);  // LA2_ERR_CUDA
        return;
    }
    const uint32_t sA = base + L::kA, sB = base + L::kB, sBlo = base + L::kBlo;
    const uint32_t sC = base + L::kC, sW = base + L::kW;
    float* pw = reinterpret_cast<float*>(smem_raw + L::kPow);
    auto bar = [&](int b) { return base + L::kBar + 8u * b; };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem_raw + L::kAbort);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int segs_in_grid = p.nseg;
    const int g = blockIdx.x % segs_in_grid;
    const int unit = blockIdx.x / segs_in_grid;  // (sequence, role)
    const int role_id = unit % p.nroles;
    const int bh = unit / p.nroles;
    const Role& R = p.role[role_id];
    const int dir = R.dir;
    const int T = p.T;
    const int nb = (T + kTB - 1) / kTB;
    // this CTA's steps (in scan order): [s0, s0 + ns)
    const int s0 = g * p.seg_tiles;
    const int ns = max(0, min(p.seg_tiles, nb - s0));
    const float lam = p.decay[bh % p.H];

    // ---- set-up
    {
        const double l2 = log2(static_cast<double>(lam));
        for (int n = tid; n <= kTB; n += kThreads) pw[n] = static_cast<float>(exp2(n * l2));
        for (uint32_t off = tid * 16; off < 2 * L::kWsz; off += kThreads * 16)
            st_shared_v4(sW + off, 0u, 0u, 0u, 0u);
    }
    if (warp == 0) {
        tmem_alloc(base + L::kTmemSlot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        const uint32_t counts[NBAR] = {1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1,
                                       256, 256, 256, 256, 256, 256, 256, 3};
        for (int b = 0; b < NBAR; ++b) mbar_init(bar(b), counts[b]);
        *abort_flag = 0;
        fence_mbar_init();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem_raw + L::kTmemSlot);
    // TMEM: S / P in two buffers (128 columns each), X in two buffers (DC each).
    // dW of tile s goes to the X buffer of tile s+1: X of tile s-1 has been read
    // out of it, and X of tile s+1 is not issued before dW has been read.
    auto tS = [&](int b) { return tmem + static_cast<uint32_t>(b * 128); };
    auto tX = [&](int b) { return tmem + 256 + static_cast<uint32_t>(b * DC); };
    auto tile_of = [&](int step) { return dir > 0 ? s0 + step : nb - 1 - (s0 + step); };
    // fp32 state slot of segment gg of this (sequence, role)
    auto seg_slot = [&](int gg) {
        return p.seg_state + (static_cast<size_t>(unit) * (p.nseg - 1) + gg) * (DA * DC);
    };

    if (warp == 0) {
        // ================================================= TMA producer
        if (lane == 0 && ns > 0) {
            prefetch_tmap(&R.ta);
            prefetch_tmap(&R.tb);
            prefetch_tmap(&R.tc);
            auto load_a = [&](int i) {
                mbar_arrive_expect_tx(bar(FULL_A), kTB * DA * 2);
                for (int g = 0; g < DA / 64; ++g)
                    tma_load_3d(sA + g * 16384, &R.ta, bar(FULL_A), g * 64, i * kTB, bh);
            };
            auto load_b = [&](int i, int slot) {
                const uint32_t b = bar(FULL_B0 + slot);
                mbar_arrive_expect_tx(b, kTB * DA * 2);
                for (int g = 0; g < DA / 64; ++g)
                    tma_load_3d(sB + slot * L::kBsz + g * 16384, &R.tb, b, g * 64, i * kTB, bh);
            };
            auto load_c = [&](int i) {
                mbar_arrive_expect_tx(bar(FULL_C), kTB * DC * 2);
                for (int g = 0; g < DC / 64; ++g)
                    tma_load_3d(sC + g * 16384, &R.tc, bar(FULL_C), g * 64, i * kTB, bh);
            };
            load_a(tile_of(0));
            load_b(tile_of(0), 0);
            if (ns > 1) load_b(tile_of(1), 1);
            load_c(tile_of(0));
            for (int s = 0; s < ns; ++s) {
                const uint32_t ph = s & 1;
                // A is free once S and X = A W of tile s are done; B buffer s % 2 once
                // dW of tile s is done; C once X += P C is done too.  Waiting in
                // this order keeps every waiter within one phase of its barrier.
                if (!wait_bar(bar(B_S0 + (s & 1)), (s >> 1) & 1, abort_flag, p.status, 13)) break;
                if (!wait_bar(bar(B_X0 + (s & 1)), (s >> 1) & 1, abort_flag, p.status, 10)) break;
                if (s + 1 < ns) load_a(tile_of(s + 1));
                if (!wait_bar(bar(B_D), ph, abort_flag, p.status, 11)) break;
                if (s + 2 < ns) load_b(tile_of(s + 2), s & 1);
                if (!wait_bar(bar(B_PC0 + (s & 1)), (s >> 1) & 1, abort_flag, p.status, 12)) break;
                if (s + 1 < ns) load_c(tile_of(s + 1));
            }
        }
    } else if (warp == 3) {
        // ================================================= MMA issuer 0
        // S of tile s into S buffer s % 2, once X += P C of tile s-2, which read
        // the P in that buffer, is done
        if (lane == 0) {
            constexpr uint32_t kIdS = idesc_bf16_f32(128, kTB, 0, 0);
            for (int s = 0; s < ns; ++s) {
                const uint32_t ph = s & 1;
                const uint32_t sBs = sB + (s & 1) * L::kBsz;
                if (!wait_bar(bar(FULL_A), ph, abort_flag, p.status, 20)) break;
                if (!wait_bar(bar(FULL_B0 + (s & 1)), (s >> 1) & 1, abort_flag, p.status, 21)) break;
                if (s > 1 &&
                    !wait_bar(bar(B_PC0 + (s & 1)), ((s - 2) >> 1) & 1, abort_flag, p.status, 22))
                    break;
                tc_fence_after();
                const uint32_t st = tS(s & 1);
#pragma unroll 1
                for (int k = 0; k < DA / 16; ++k) {
                    const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
                    mma_bf16_ss(st, sdesc_sw128(sA + off, 16, 1024), sdesc_sw128(sBs + off, 16, 1024),
                                kIdS, k > 0);
                }
                mma_commit(bar(B_S0 + (s & 1)));
            }
            mma_commit(bar(B_FIN));
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer 1
        // X += P C of tile s, P read from S buffer s % 2
        if (lane == 0) {
            constexpr uint32_t kIdX = idesc_bf16_f32(128, DC, 0, 1);
            for (int s = 0; s < ns; ++s) {
                const uint32_t ph = s & 1;
                if (!wait_bar(bar(B_P0 + (s & 1)), (s >> 1) & 1, abort_flag, p.status, 23)) break;
                if (!wait_bar(bar(B_XS), ph, abort_flag, p.status, 24)) break;
                if (!wait_bar(bar(FULL_C), ph, abort_flag, p.status, 25)) break;
                tc_fence_after();
                const uint32_t xt = tX(s & 1), st = tS(s & 1);
#pragma unroll 1
                for (int k = 0; k < kTB / 16; ++k) {
                    const uint64_t cdesc = sdesc_sw128(sC + k * 2048, 16384, 1024);
                    mma_bf16_ts(xt, st + k * 16, cdesc, kIdX, 1);
                    mma_bf16_ts(xt, st + k * 16 + 8, cdesc, kIdX, 1);
                }
                mma_commit(bar(B_PC0 + (s & 1)));
            }
            mma_commit(bar(B_FIN));
        }
    } else if (warp == 2) {
        // ================================================= MMA issuer 2
        // X = A hi(W) + A lo(W) into X buffer s % 2, then dW into X buffer (s+1) % 2
        if (lane == 0) {
            constexpr uint32_t kIdX = idesc_bf16_f32(128, DC, 0, 1);
            constexpr uint32_t kIdW = idesc_bf16_f32(DA, DC, 1, 1);
            for (int s = 0; s < ns; ++s) {
                const uint32_t ph = s & 1;
                const uint32_t sBs = sB + (s & 1) * L::kBsz;
                // B_WR completes once when the epilogue has set the initial state
                // and once per tile when it has updated W and read dW (which sat
                // in X buffer s % 2)
                {
                    if (!wait_bar(bar(B_WR), ph, abort_flag, p.status, 30)) break;
                    if (!wait_bar(bar(FULL_A), ph, abort_flag, p.status, 34)) break;
                    tc_fence_after();
                    const uint32_t xt = tX(s & 1);
#pragma unroll 1
                    for (int k = 0; k < DA / 16; ++k) {
                        const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
                        const uint64_t adesc = sdesc_sw128(sA + off, 16, 1024);
                        mma_bf16_ss(xt, adesc, sdesc_sw128(sW + k * 2048, DA * 128, 1024), kIdX, k > 0);
                        mma_bf16_ss(xt, adesc, sdesc_sw128(sW + L::kWsz + k * 2048, DA * 128, 1024),
                                    kIdX, 1);
                    }
                    mma_commit(bar(B_X0 + (s & 1)));
                }
                if (!wait_bar(bar(B_BS), ph, abort_flag, p.status, 31)) break;
                if (!wait_bar(bar(FULL_C), ph, abort_flag, p.status, 32)) break;
                // X buffer (s+1) % 2 was read out after tile s-1
                if (s > 0 &&
                    !wait_bar(bar(B_XF0 + ((s + 1) & 1)), ((s - 1) >> 1) & 1, abort_flag, p.status, 33))
                    break;
                tc_fence_after();
                const uint32_t dt = tX((s + 1) & 1);
#pragma unroll 1
                for (int k = 0; k < kTB / 16; ++k) {
                    const uint64_t cdesc = sdesc_sw128(sC + k * 2048, 16384, 1024);
                    mma_bf16_ss(dt, sdesc_sw128(sBs + k * 2048, 16384, 1024), cdesc, kIdW, k > 0);
                    mma_bf16_ss(dt, sdesc_sw128(sBlo + k * 2048, 16384, 1024), cdesc, kIdW, 1);
                }
                mma_commit(bar(B_D));
            }
            mma_commit(bar(B_FIN));
        }
    } else if (warp >= 4 && warp < 12) {
        // ================================================= mask group
        // two warps per lane quadrant; warp part p takes the 16-column groups
        // g with g % 2 == p, which splits the causal triangle's work evenly
        const int quad = warp & 3, part = (warp - 4) >> 2;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const float ws = dir > 0 ? pw[kTB - 1 - r] : pw[r];
        for (int s = 0; s < ns; ++s) {
            const uint32_t ph = s & 1;
            if (!wait_bar(bar(B_S0 + (s & 1)), (s >> 1) & 1, abort_flag, p.status, 40)) break;
            const uint32_t st = tS(s & 1);
            tc_fence_after();
            // row r of w_s B (S, which reads B unscaled, is done): hi in place,
            // lo into its own buffer once the previous tile's dW, its only
            // reader, is done.  Part p does the chunks of half p of the row.
            if (s > 0 && !wait_bar(bar(B_D), ph ^ 1, abort_flag, p.status, 41)) break;
            const uint32_t sBs = sB + (s & 1) * L::kBsz;
#pragma unroll
            for (int k = 0; k < DA / 16; ++k) {
                const int chunk = part * (DA / 16) + k;
                const uint32_t off = (chunk >> 3) * 16384 + sw128(r, chunk & 7);
                uint32_t v[4], h[4], l[4];
                ld_shared_v4(sBs + off, v[0], v[1], v[2], v[3]);
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    split_pack2(bf16lo_to_f32(v[u]) * ws, bf16hi_to_f32(v[u]) * ws, h[u], l[u]);
                st_shared_v4(sBs + off, h[0], h[1], h[2], h[3]);
                st_shared_v4(sBlo + off, l[0], l[1], l[2], l[3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(bar(B_BS));
            {
            // P = decay-masked S, hi + lo bf16, over the 16 columns of S each
            // group of 16 came from: [hi (8 cols) | lo (8 cols)], the A-operand
            // layout of one K = 16 step.  Every group is loaded before it is
            // overwritten, also groups the mask zeroes entirely: storing over S
            // columns that were not read first made the following TMEM-operand
            // MMAs about 10x slower.
            // Part p takes the 32-column pairs of groups {4k + 2p, 4k + 2p + 1},
            // which splits the causal triangle's work about evenly.
#pragma unroll 1
            for (int pr = part; pr < kTB / 32; pr += 2) {
                float sv[32];
                tmem_ld32(st + lane_off + pr * 32, sv);
                uint32_t pk[32];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int grp = 2 * pr + h2;
                    const int lo_g = 2 * quad, hi_g = 2 * quad + 1;
                    const int kind = (grp == lo_g || grp == hi_g) ? 1 : ((dir > 0) == (grp < lo_g) ? 2 : 0);
                    if (kind == 2) {
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int c0 = grp * 16 + 2 * u;
                            const float p0 = sv[16 * h2 + 2 * u] * pw[dir > 0 ? r - c0 : c0 - r];
                            const float p1 = sv[16 * h2 + 2 * u + 1] * pw[dir > 0 ? r - c0 - 1 : c0 + 1 - r];
                            split_pack2(p0, p1, pk[16 * h2 + u], pk[16 * h2 + 8 + u]);
                        }
                    } else if (kind == 1) {
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int c0 = grp * 16 + 2 * u;
                            const int lag0 = dir > 0 ? r - c0 : c0 - r;
                            const int lag1 = dir > 0 ? r - c0 - 1 : c0 + 1 - r;
                            const float p0 = lag0 >= 0 ? sv[16 * h2 + 2 * u] * pw[lag0 < 0 ? 0 : lag0] : 0.f;
                            const float p1 =
                                lag1 >= 0 ? sv[16 * h2 + 2 * u + 1] * pw[lag1 < 0 ? 0 : lag1] : 0.f;
                            split_pack2(p0, p1, pk[16 * h2 + u], pk[16 * h2 + 8 + u]);
                        }
                    } else {
#pragma unroll
                        for (int u = 0; u < 16; ++u) pk[16 * h2 + u] = 0u;
                    }
                }
                tmem_st32u(st + lane_off + pr * 32, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(B_P0 + (s & 1)));
            }
        }
    } else if (warp >= 12) {
        // ================================================= epilogue group
        const int quad = warp & 3, half = (warp - 12) >> 2;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        constexpr int kCols = DC / 2;                 // columns of X and W this thread handles
        const int c0 = half * kCols;
        const float wx = dir > 0 ? pw[r + 1] : pw[kTB - r];
        const float lamTB = pw[kTB];
        const bool owns_w_row = (DA == 128) || (lane < 16);
        const int wrow = (DA == 128) ? r : quad * 16 + (lane & 15);
        {
            // initial state of this segment, W_in(g) = f W_in(g-1) + S_{g-1} with
            // f = lambda^(T_B n), as its hi/lo bf16 pair (zero for the first)
            if (g > 0 && owns_w_row) {
                const float f = static_cast<float>(
                    exp2(static_cast<double>(kTB) * p.seg_tiles * log2(static_cast<double>(lam))));
#pragma unroll 1
                for (int k = 0; k < kCols / 16; ++k) {
                    const uint32_t col = c0 + k * 16;
                    float w[16];
#pragma unroll
                    for (int u = 0; u < 16; ++u) w[u] = 0.f;
                    for (int gp = 0; gp < g; ++gp) {
                        const float* src = seg_slot(gp) + static_cast<size_t>(wrow) * DC + col;
#pragma unroll
                        for (int u = 0; u < 16; ++u) w[u] = fmaf(f, w[u], src[u]);
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
            }
            fence_proxy_async_smem();
            mbar_arrive(bar(B_WR));
            float* xg = R.x + static_cast<size_t>(bh) * T * DC;
            const int grp = lane >> 3, j = lane & 7;
            for (int s = 0; s < ns; ++s) {
                const uint32_t ph = s & 1;
                const int i = tile_of(s);
                const uint32_t xt = tX(s & 1);
                // X row r *= w_x(r)   (the inter-tile term, still alone in X)
                if (!wait_bar(bar(B_X0 + (s & 1)), (s >> 1) & 1, abort_flag, p.status, 50)) break;
                tc_fence_after();
#pragma unroll 1
                for (int k = 0; k < kCols / 32; ++k) {
                    float x[32];
                    const uint32_t col = c0 + k * 32;
                    tmem_ld32(xt + lane_off + col, x);
#pragma unroll
                    for (int u = 0; u < 32; ++u) x[u] *= wx;
                    tmem_st32(xt + lane_off + col, x);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(B_XS));
                // W <- lambda^T_B W + dW.  The state is kept as its hi + lo bf16
                // pair (a 16-bit significand, ~2^-17 relative per update), which
                // is also the next tile's MMA operand; X = A W of this tile, which
                // read it, is done.
                if (!wait_bar(bar(B_D), ph, abort_flag, p.status, 51)) break;
                tc_fence_after();
#pragma unroll 1
                for (int k = 0; k < kCols / 32; ++k) {
                    float d[32];
                    tmem_ld32(tX((s + 1) & 1) + lane_off + c0 + k * 32, d);
                    if (owns_w_row) {
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const uint32_t col = c0 + k * 32 + hh * 16;
                            const uint32_t grpo = (col >> 6) * (DA * 128);
                            const int q = (col & 63) >> 3;
                            const uint32_t a0 = sW + grpo + sw128(wrow, q);
                            const uint32_t a1 = sW + grpo + sw128(wrow, q + 1);
                            uint32_t h[8], l[8];
                            ld_shared_v4(a0, h[0], h[1], h[2], h[3]);
                            ld_shared_v4(a1, h[4], h[5], h[6], h[7]);
                            ld_shared_v4(a0 + L::kWsz, l[0], l[1], l[2], l[3]);
                            ld_shared_v4(a1 + L::kWsz, l[4], l[5], l[6], l[7]);
#pragma unroll
                            for (int z = 0; z < 8; ++z) {
                                const float w0 = fmaf(lamTB, bf16lo_to_f32(h[z]) + bf16lo_to_f32(l[z]),
                                                      d[16 * hh + 2 * z]);
                                const float w1 = fmaf(lamTB, bf16hi_to_f32(h[z]) + bf16hi_to_f32(l[z]),
                                                      d[16 * hh + 2 * z + 1]);
                                split_pack2(w0, w1, h[z], l[z]);
                            }
                            st_shared_v4(a0, h[0], h[1], h[2], h[3]);
                            st_shared_v4(a1, h[4], h[5], h[6], h[7]);
                            st_shared_v4(a0 + L::kWsz, l[0], l[1], l[2], l[3]);
                            st_shared_v4(a1 + L::kWsz, l[4], l[5], l[6], l[7]);
                        }
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(bar(B_WR));
                // X of tile i, 32 columns at a time: TMEM -> registers, then an
                // 8 x 8 transpose of float4s among each group of 8 lanes (warp
                // shuffles), after which every store instruction writes four whole
                // 128-byte rows.  The X buffer is released once read.
                if (!wait_bar(bar(B_PC0 + (s & 1)), (s >> 1) & 1, abort_flag, p.status, 52)) break;
                tc_fence_after();
#pragma unroll 1
                for (int b = 0; b < kCols / 32; ++b) {
                    float v[32];
                    tmem_ld32(xt + lane_off + c0 + 32 * b, v);
                    if (b == kCols / 32 - 1) {
                        tc_fence_before();
                        mbar_arrive(bar(B_XF0 + (s & 1)));
                    }
                    // lane j of a group holds chunk c (4 floats) of its row in
                    // v[4c..4c+3]; afterwards chunk j of row 8*grp + c
#pragma unroll
                    for (int st = 4; st >= 1; st >>= 1) {
                        const bool up = (j & st) != 0;
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            if (c & st) continue;
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float send = up ? v[4 * c + e] : v[4 * (c | st) + e];
                                const float recv = __shfl_xor_sync(0xffffffffu, send, st);
                                if (up) v[4 * c + e] = recv;
                                else v[4 * (c | st) + e] = recv;
                            }
                        }
                    }
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const int row = i * kTB + quad * 32 + grp * 8 + c;
                        if (row < T)
                            st_global_v4(xg + static_cast<size_t>(row) * DC + c0 + 32 * b + 4 * j,
                                         v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                    }
                }
            }
        }
    }

    // ---- tear-down: wait (bounded) until both issuers' MMAs are done, free TMEM
    __syncthreads();
    if (tid == 32 && ns > 0) {
        if (!mbar_wait(bar(B_FIN), 0)) atomicCAS(p.status, 0, 5 | (60 << 8));
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}


// ---------------------------------------------------------------------------
// State pre-pass for segmented sequences.  One CTA per (sequence, role,
// segment but the last).  The state a segment of n tiles leaves behind when it
// starts from zero is
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
    const int segs_in_grid = p.nseg - 1;
    const int g = blockIdx.x % segs_in_grid;
    const int unit = blockIdx.x / segs_in_grid;
    const int role_id = unit % p.nroles;
    const int bh = unit / p.nroles;
    const Role& R = p.role[role_id];
    const int dir = R.dir;
    const int nb = (p.T + kTB - 1) / kTB;
    const int s0 = g * p.seg_tiles;
    const int ns = max(0, min(p.seg_tiles, nb - s0));
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
                    tma_load_3d(sB + slot * L::kBsz + gg * 16384, &R.tb, bb, gg * 64, i * kTB, bh);
                mbar_arrive_expect_tx(bc, kTB * DC * 2);
                for (int gg = 0; gg < DC / 64; ++gg)
                    tma_load_3d(sC + slot * L::kCsz + gg * 16384, &R.tc, bc, gg * 64, i * kTB, bh);
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
            const float wt = static_cast<float>(exp2(static_cast<double>(e) * l2));
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
            float* dst0 = p.seg_state + (static_cast<size_t>(unit) * (p.nseg - 1) + g) * (DA * DC) +
                          static_cast<size_t>(srow) * DC;
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
