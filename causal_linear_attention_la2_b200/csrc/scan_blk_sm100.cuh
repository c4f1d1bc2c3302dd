// scan_blk_sm100.cuh -- bf16-input tcgen05 scan for the tile lengths T_B = 64
// and T_B = 256 of the Lightning Attention-2 tiling ("Lightning Attention"
// page, lizeman.github.io llm-arch-kb, section 2 steps 1-4; its section 4
// reports block sizes 64, 128 and 256 swept, 128 best on A100 and 256 on
// H100).  The same decayed scan as scan_ws_sm100.cuh,
//
//   dir = +1:  x_t = sum_{s<=t} lambda^(t-s) (a_t . b_s) c_s
//   dir = -1:  x_t = sum_{s>=t} lambda^(s-t) (a_t . b_s) c_s
//
// but with the state carried across blocks of 64 or 256 rows.  The tensor-core
// tile is 128 rows (MMA M = 128), so
//
// - T_B = 256: a block is a pair of 128-row tiles u0, u1 (in scan order).  Its
//   intra-block part is three 128 x 128 score blocks, S_00 = A_0 B_0^T and
//   S_11 = A_1 B_1^T with the causal decay mask and S_10 = A_1 B_0^T whole
//   (weights lambda^(128 + lag)), so X_1 gains P_10 C_0 + P_11 C_1; both
//   tiles read the state of the block's start (row weights lambda^(rho+1)
//   resp. lambda^(256-rho) on block row rho), and the state is updated once
//   per block: W <- lambda^256 W + sum_rho w_s(rho) b_rho c_rho^T.
// - T_B = 64: a 128-row tile holds two blocks f, s (in scan order).  P keeps
//   only the two 64 x 64 diagonal blocks; the rows of f read the state W of the
//   tile's start, the rows of s the state after f,
//   W_mid = lambda^64 W + dW_f, and the tile ends with W <- lambda^64 W_mid + dW_s.
//
// One CTA per (sequence, role, 64 value columns): a 256-row block needs A, both
// B tiles, the lo part of w_s B, both C tiles and the state's hi/lo pair at once
// (192 KB at d = 128 with 64 value columns), and three S blocks plus two X
// accumulators fill the 512 TMEM columns.  The phases run one after the other
// (TMA, then MMAs issued by one thread, then all warps on TMEM and shared
// memory), every hand-off an mbarrier or a block barrier: simple and exact, not
// overlapped like the T_B = 128 kernel.  Operands the kernel forms (P, w_s B,
// the state) enter the tensor cores as bf16 hi + lo pairs; the state is kept in
// fp32 registers.  Carried states as in the T_B = 128 kernel (ws::Role): an
// initial state (forward: before position 0; reverse: entering at position
// T-1, so the reverse scan's first block weighs it by lambda^(n-1-r) over its
// n rows and decays it by lambda^(n-1)), read transposed with init_t; the
// final state (forward: after position T-1, the last block's update using its
// true row count; reverse: lambda times the state at position 0); and the
// per-position factor colf of the normalised form.  No segments.
#pragma once
#include "ptx_sm100.cuh"
#include "scan_ws_sm100.cuh"

namespace la2 {
namespace blk {

constexpr int kThreads = 256;
constexpr int kDC = 64;  // value columns per CTA

struct Params {
    ws::Role role[3];    // maps, output, direction, carried states and per-position factor
    const float* decay;  // [H]
    int* status;         // device status word
    int H, T, nroles, bthd;
    int dc;              // the group's full value width (row length of the outputs)
    int nslice;          // dc / 64: CTAs per (sequence, role)
    int xbf16;           // 1: outputs bf16 (rounded to nearest even once), 0: fp32
};

template <int DA, int TB>
struct Smem {
    static constexpr uint32_t kAsz = 128 * DA * 2;   // a 128-row A (or B) tile
    static constexpr uint32_t kCsz = 128 * kDC * 2;  // a 128-row, 64-column C tile
    static constexpr uint32_t kWsz = DA * kDC * 2;   // hi(W) or lo(W)
    static constexpr int NB = TB == 256 ? 2 : 1;
    static constexpr uint32_t kA = 0;
    static constexpr uint32_t kB = kA + kAsz;            // B tiles (then hi(w_s B) in place)
    static constexpr uint32_t kLo = kB + NB * kAsz;      // lo(w_s B)
    static constexpr uint32_t kC = kLo + kAsz;           // C tiles
    static constexpr uint32_t kW = kC + NB * kCsz;       // W: hi, lo
    static constexpr uint32_t kW2 = kW + 2 * kWsz;       // T_B = 64: W_mid: hi, lo
    static constexpr uint32_t kPow = kW2 + (TB == 64 ? 2 * kWsz : 0);  // lambda^n, n = 0..256
    static constexpr uint32_t kBar = kPow + 1088;
    static constexpr uint32_t kTmemSlot = kBar + 16;
    static constexpr uint32_t kAbort = kTmemSlot + 4;
    static constexpr uint32_t kBytes = kAbort + 12;
    static_assert(kBytes <= 232448, "shared memory over the 227 KB per-CTA limit");
};

template <int DA, int TB>
__global__ void __launch_bounds__(kThreads, 1)
la2_scan_blk(const __grid_constant__ Params p)
{
    static_assert(DA == 64 || DA == 128, "DA in {64, 128}");
    static_assert(TB == 64 || TB == 256, "T_B in {64, 256}");
    using L = Smem<DA, TB>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    if (base & 1023u) {
        if (threadIdx.x == 0) atomicCAS(p.status, 0, 4);
        return;
    }
    const uint32_t sA = base + L::kA, sB = base + L::kB, sLo = base + L::kLo, sC = base + L::kC;
    const uint32_t sW = base + L::kW, sW2 = base + L::kW2;
    float* pw = reinterpret_cast<float*>(smem_raw + L::kPow);
    const uint32_t barT = base + L::kBar, barM = base + L::kBar + 8;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem_raw + L::kAbort);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int unit = blockIdx.x / p.nslice, cs = blockIdx.x % p.nslice;
    const int role_id = unit % p.nroles, bh = unit / p.nroles;
    const ws::Role& R = p.role[role_id];
    const int dir = R.dir, T = p.T;
    const int nb = (T + 127) / 128;  // 128-row tiles
    const float lam = p.decay[bh % p.H];

    if (warp == 0) {
        tmem_alloc(base + L::kTmemSlot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(barT, 1);
        mbar_init(barM, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    {
        const double l2 = log2(static_cast<double>(lam));
        for (int n = tid; n <= 256; n += kThreads) pw[n] = static_cast<float>(exp2(n * l2));
        const uint32_t wbytes = (TB == 64 ? 4 : 2) * L::kWsz;  // W (and W_mid) = 0
        for (uint32_t off = tid * 16; off < wbytes; off += kThreads * 16) st_shared_v4(sW + off, 0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem_raw + L::kTmemSlot);

    // thread roles in the all-warp phases: TMEM lane quadrant q, column half hf
    const int quad = warp & 3, hf = warp >> 2;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    // the state rows this thread owns (dW's TMEM layout: M = 128 one row per
    // lane; M = 64 rows 16q .. 16q+15 in lanes 0..15 of quadrant q)
    const bool owns_w_row = (DA == 128) || (lane < 16);
    const int wrow = (DA == 128) ? r : quad * 16 + (lane & 15);
    float wreg[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) wreg[u] = 0.f;

    // output rows: [B, H, T, dc] (row stride dc) or [B, T, H, dc] (stride H dc)
    const size_t xrs = p.bthd ? static_cast<size_t>(p.H) * p.dc : static_cast<size_t>(p.dc);
    const size_t xoff = (p.bthd ? (static_cast<size_t>(bh / p.H) * T * p.H + bh % p.H) * p.dc
                                : static_cast<size_t>(bh) * T * p.dc) + kDC * cs;
    const bool xb16 = p.xbf16 != 0;
    char* const xg = static_cast<char*>(R.x) + xoff * (xb16 ? 2 : 4);

    constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t kIdX = idesc_bf16_f32(128, kDC, 0, 1);
    constexpr uint32_t kIdW = idesc_bf16_f32(DA, kDC, 1, 1);
    const uint64_t dA = sdesc_sw128(sA, 16, 1024);

    uint32_t phT = 0, phM = 0;
    bool ok = true;
    auto wait_t = [&](int site) {
        ok = ok && ws::wait_bar(barT, phT, abort_flag, p.status, site);
        phT ^= 1u;
    };
    auto wait_m = [&](int site) {
        ok = ok && ws::wait_bar(barM, phM, abort_flag, p.status, site);
        phM ^= 1u;
        tc_fence_after();
    };
    auto load_tile = [&](uint32_t dst, const CUtensorMap* map, int tile, int cols, int x0) {
        for (int gg = 0; gg < cols / 64; ++gg)
            ws::load_box(dst + gg * 16384, map, barT, x0 + gg * 64, tile * 128, bh, p.H, p.bthd);
    };
    // an L2 prefetch of a tile that a later phase loads (the phases do not
    // overlap, so without it every load would wait for HBM)
    auto prefetch_tile = [&](const CUtensorMap* map, int tile, int cols, int x0) {
        if (tile < 0 || tile * 128 >= T) return;
        for (int gg = 0; gg < cols / 64; ++gg) ws::prefetch_box(map, x0 + gg * 64, tile * 128, bh, p.H, p.bthd);
    };
    // S (128 x 128, fp32) = A B^T into TMEM column t
    auto mma_s = [&](uint32_t t, uint32_t sb) {
        const uint64_t db = sdesc_sw128(sb, 16, 1024);
#pragma unroll
        for (int k = 0; k < DA / 16; ++k) {
            const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
            mma_bf16_ss(t, desc_add(dA, off), desc_add(db, off), kIdS, k > 0);
        }
    };
    // X (128 x 64) = A hi(W) + A lo(W), W at sw
    auto mma_xw = [&](uint32_t t, uint32_t sw) {
        const uint64_t dw = sdesc_sw128(sw, DA * 128, 1024);
#pragma unroll
        for (int k = 0; k < DA / 16; ++k) {
            const uint64_t ad = desc_add(dA, (k >> 2) * 16384 + (k & 3) * 32);
            mma_bf16_ss(t, ad, desc_add(dw, k * 2048), kIdX, k > 0);
            mma_bf16_ss(t, ad, desc_add(dw, L::kWsz + k * 2048), kIdX, 1);
        }
    };
    // X += P C, P the hi/lo pairs in TMEM at tp, C at sc
    auto mma_pc = [&](uint32_t t, uint32_t tp, uint32_t sc, bool first) {
        const uint64_t dc = sdesc_sw128(sc, 16384, 1024);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const uint64_t cd = desc_add(dc, k * 2048);
            mma_bf16_ts_w(t, tp + k * 16, cd, kIdX, (first && k == 0) ? 0u : 1u, 1u);
            mma_bf16_ts_w(t, tp + k * 16 + 8, cd, kIdX, 1u, 1u);
        }
    };
    // dW (+)= (w_s B)^T C over K steps [k0, k1) of 16 rows: hi (in the B
    // tile) and lo parts of w_s B
    auto mma_dw = [&](uint32_t t, uint32_t sb, uint32_t sc, int k0, int k1, bool first) {
        const uint64_t db = sdesc_sw128(sb, 16384, 1024), dl = sdesc_sw128(sLo, 16384, 1024);
        const uint64_t dc = sdesc_sw128(sc, 16384, 1024);
        for (int k = k0; k < k1; ++k) {
            const uint64_t cd = desc_add(dc, k * 2048);
            mma_bf16_ss(t, desc_add(db, k * 2048), cd, kIdW, (first && k == k0) ? 0u : 1u);
            mma_bf16_ss(t, desc_add(dl, k * 2048), cd, kIdW, 1u);
        }
    };
    // the per-position factor f on the summed position (the normalised form's
    // backward; null elsewhere): x_t = sum_s lambda^|t-s| (a_t . b_s) f_s c_s,
    // applied to P's columns and to the state-update weights of the keys
    const float* colf = R.colf ? R.colf + static_cast<size_t>(bh) * T : nullptr;
    auto f_at = [&](int tile, int row) -> float {
        const int t = tile * 128 + row;
        return t < T ? __ldg(colf + t) : 0.f;
    };
    // P from the S block at t, whose columns are the keys of tile ktile:
    // weight(row, col) per element (0 off the mask), times f of the key with
    // colf, stored back as [hi (8 columns) | lo (8 columns)] per 16 columns
    auto make_p = [&](uint32_t t, int ktile, auto weight) {
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
            const int col0 = 64 * hf + 32 * cc;
            float sv[32];
            tmem_ld32(t + lane_off + col0, sv);
#pragma unroll
            for (int u = 0; u < 32; ++u) sv[u] *= weight(r, col0 + u);
            if (colf) {
#pragma unroll
                for (int u = 0; u < 32; ++u) sv[u] *= f_at(ktile, col0 + u);
            }
            uint32_t pk[32];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    split_pack2v(make_float2(sv[16 * h2 + 2 * u], sv[16 * h2 + 2 * u + 1]), pk[16 * h2 + u],
                                 pk[16 * h2 + 8 + u]);
            tmem_st32u(t + lane_off + col0, pk);
        }
    };
    // hi(w_s B) in place and lo(w_s B) into sLo, row r's weight w, times f
    // of that key (tile ktile) with colf (this thread: half hf of the row's
    // 16-byte chunks)
    auto split_b = [&](uint32_t sb, int ktile, float w) {
        if (colf) w *= f_at(ktile, r);
#pragma unroll
        for (int k = 0; k < DA / 16; ++k) {
            const int chunk = hf * (DA / 16) + k;
            const uint32_t off = (chunk >> 3) * 16384 + ws::sw128(r, chunk & 7);
            uint32_t v[4], h[4], l[4];
            ld_shared_v4(sb + off, v[0], v[1], v[2], v[3]);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                split_pack2v(mul2(make_float2(bf16lo_to_f32(v[u]), bf16hi_to_f32(v[u])), make_float2(w, w)), h[u],
                             l[u]);
            st_shared_v4(sb + off, h[0], h[1], h[2], h[3]);
            st_shared_v4(sLo + off, l[0], l[1], l[2], l[3]);
        }
    };
    // W <- f W + dW (dW in TMEM at t; d = null: W <- f W): the fp32 state in
    // registers, its hi/lo pair to sw (the next A W MMA's operand)
    auto update_w = [&](uint32_t t, float f, uint32_t sw) {
        float d[32];
        tmem_ld32(t + lane_off + 32 * hf, d);
        if (owns_w_row) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int col = 32 * hf + 16 * hh;
                const uint32_t o0 = ws::sw128(wrow, col >> 3), o1 = ws::sw128(wrow, (col >> 3) + 1);
                uint32_t h[8], l[8];
#pragma unroll
                for (int z = 0; z < 8; ++z) {
                    const int u = 16 * hh + 2 * z;
                    const float2 w = fma2(make_float2(f, f), make_float2(wreg[u], wreg[u + 1]),
                                          make_float2(d[u], d[u + 1]));
                    wreg[u] = w.x;
                    wreg[u + 1] = w.y;
                    split_pack2v(w, h[z], l[z]);
                }
                st_shared_v4(sw + o0, h[0], h[1], h[2], h[3]);
                st_shared_v4(sw + o1, h[4], h[5], h[6], h[7]);
                st_shared_v4(sw + L::kWsz + o0, l[0], l[1], l[2], l[3]);
                st_shared_v4(sw + L::kWsz + o1, l[4], l[5], l[6], l[7]);
            }
        }
    };
    // W <- f W without a dW (the hi/lo pair rewritten from the registers)
    auto scale_w = [&](float f, uint32_t sw) {
        if (owns_w_row) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int col = 32 * hf + 16 * hh;
                const uint32_t o0 = ws::sw128(wrow, col >> 3), o1 = ws::sw128(wrow, (col >> 3) + 1);
                uint32_t h[8], l[8];
#pragma unroll
                for (int z = 0; z < 8; ++z) {
                    const int u = 16 * hh + 2 * z;
                    wreg[u] *= f;
                    wreg[u + 1] *= f;
                    split_pack2v(make_float2(wreg[u], wreg[u + 1]), h[z], l[z]);
                }
                st_shared_v4(sw + o0, h[0], h[1], h[2], h[3]);
                st_shared_v4(sw + o1, h[4], h[5], h[6], h[7]);
                st_shared_v4(sw + L::kWsz + o0, l[0], l[1], l[2], l[3]);
                st_shared_v4(sw + L::kWsz + o1, l[4], l[5], l[6], l[7]);
            }
        }
    };
    // 32 columns of X at t (plus f times Y at ty, when ty != 0) for row r of
    // tile `tile`, written to the output
    auto store_x = [&](uint32_t t, uint32_t ty, float f, int tile) {
        float v[32];
        tmem_ld32(t + lane_off + 32 * hf, v);
        if (ty != 0u) {
            float y[32];
            tmem_ld32(ty + lane_off + 32 * hf, y);
#pragma unroll
            for (int u = 0; u < 32; ++u) v[u] = fmaf(f, y[u], v[u]);
        }
        const int row = tile * 128 + r;
        if (row < T && xb16) {
            uint16_t* dst = reinterpret_cast<uint16_t*>(xg) + static_cast<size_t>(row) * xrs + 32 * hf;
#pragma unroll
            for (int u = 0; u < 32; u += 8)
                st_global_v4_b32(dst + u, pack_bf16x2(v[u], v[u + 1]), pack_bf16x2(v[u + 2], v[u + 3]),
                                 pack_bf16x2(v[u + 4], v[u + 5]), pack_bf16x2(v[u + 6], v[u + 7]));
        } else if (row < T) {
            float* dst = reinterpret_cast<float*>(xg) + static_cast<size_t>(row) * xrs + 32 * hf;
#pragma unroll
            for (int u = 0; u < 32; u += 4) st_global_v4(dst + u, v[u], v[u + 1], v[u + 2], v[u + 3]);
        }
    };
    auto scale_x = [&](uint32_t t, float f) {
        float v[32];
        tmem_ld32(t + lane_off + 32 * hf, v);
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] *= f;
        tmem_st32(t + lane_off + 32 * hf, v);
    };
    auto sync_tmem = [&]() {
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    };

    // the initial state of this CTA's 64 value columns: row wrow, columns
    // 64 cs + 32 hf + u of [DA][dc] (or of [dc][DA] with init_t)
    if (R.init != nullptr) {
        if (owns_w_row) {
            const float* w0 = R.init + static_cast<size_t>(bh) * (DA * p.dc);
            const int c0 = kDC * cs + 32 * hf;
#pragma unroll
            for (int u = 0; u < 32; ++u)
                wreg[u] = R.init_t ? w0[static_cast<size_t>(c0 + u) * DA + wrow]
                                   : w0[static_cast<size_t>(wrow) * p.dc + c0 + u];
        }
        scale_w(1.f, sW);
        sync_tmem();
    }

    if constexpr (TB == 256) {
        const uint32_t tS0 = tmem, tS1 = tmem + 128, tS2 = tmem + 256, tX0 = tmem + 384, tX1 = tmem + 448;
        const uint32_t tD = tmem;  // dW reuses S_00's columns once P_00 C_0 is done
        const int nblk = (nb + 1) / 2;
        const uint32_t sB0 = sB, sB1 = sB + L::kAsz, sC0 = sC, sC1 = sC + L::kCsz;
        // rows of the sequence's last block (1..256): the forward scan's last
        // update and the reverse scan's first block use them
        const int nrow = T - 256 * (nblk - 1);
        for (int step = 0; step < nblk && ok; ++step) {
            const int m = dir > 0 ? step : nblk - 1 - step;
            const int u0 = dir > 0 ? 2 * m : 2 * m + 1, u1 = dir > 0 ? 2 * m + 1 : 2 * m;
            const bool lastf = dir > 0 && step == nblk - 1;  // state after position T-1
            const bool firstr = dir < 0 && step == 0;        // state entering at position T-1
            // B, C of both tiles and A of u0 (tiles past T read as zero)
            if (tid == 0) {
                mbar_arrive_expect_tx(barT, 3 * L::kAsz + 2 * L::kCsz);
                load_tile(sB0, &R.tb, u0, DA, 0);
                load_tile(sB1, &R.tb, u1, DA, 0);
                load_tile(sC0, &R.tc, u0, kDC, kDC * cs);
                load_tile(sC1, &R.tc, u1, kDC, kDC * cs);
                load_tile(sA, &R.ta, u0, DA, 0);
                // A of u1 (loaded after the first MMAs) and the next block's tiles
                prefetch_tile(&R.ta, u1, DA, 0);
                if (step + 1 < nblk) {
                    const int m2 = dir > 0 ? step + 1 : nblk - 2 - step;
                    for (int uu = 2 * m2; uu < 2 * m2 + 2; ++uu) {
                        prefetch_tile(&R.tb, uu, DA, 0);
                        prefetch_tile(&R.tc, uu, kDC, kDC * cs);
                        prefetch_tile(&R.ta, uu, DA, 0);
                    }
                }
            }
            wait_t(81);
            if (tid == 0) {
                mma_s(tS0, sB0);
                mma_xw(tX0, sW);
                mma_commit(barM);
            }
            wait_m(82);
            // A of u1 into the same buffer
            if (tid == 0 && ok) {
                mbar_arrive_expect_tx(barT, L::kAsz);
                load_tile(sA, &R.ta, u1, DA, 0);
            }
            wait_t(83);
            if (tid == 0 && ok) {
                mma_s(tS1, sB0);
                mma_s(tS2, sB1);
                mma_xw(tX1, sW);
                mma_commit(barM);
            }
            wait_m(84);
            if (!ok) break;
            // P_00, P_10, P_11 and the row weights of the state term
            auto diag = [&](int rr, int c) -> float {
                return dir > 0 ? (c <= rr ? pw[rr - c] : 0.f) : (c >= rr ? pw[c - rr] : 0.f);
            };
            auto off = [&](int rr, int c) -> float { return dir > 0 ? pw[128 + rr - c] : pw[128 + c - rr]; };
            make_p(tS0, u0, diag);
            make_p(tS1, u0, off);
            make_p(tS2, u1, diag);
            // rows of the reverse scan's first block weigh the entering state by
            // lambda^(n-1-j) (block row j < n), not lambda^(256-j)
            scale_x(tX0, dir > 0 ? pw[r + 1]
                                 : (firstr ? (128 + r < nrow ? pw[nrow - 1 - 128 - r] : 0.f) : pw[128 - r]));
            scale_x(tX1, dir > 0 ? pw[128 + r + 1] : (firstr ? (r < nrow ? pw[nrow - 1 - r] : 0.f) : pw[256 - r]));
            sync_tmem();
            if (tid == 0) {
                mma_pc(tX0, tS0, sC0, false);
                mma_pc(tX1, tS1, sC0, false);
                mma_pc(tX1, tS2, sC1, false);
                mma_commit(barM);
            }
            wait_m(85);
            if (!ok) break;
            store_x(tX0, 0u, 0.f, u0);
            store_x(tX1, 0u, 0.f, u1);
            // dW over the block: rows of u0 weigh lambda^(255-c) (fwd) or
            // lambda^(128+c) (rev), rows of u1 lambda^(127-c) resp. lambda^c;
            // the forward scan's last block, n rows, lambda^(n-1-j) for block
            // row j < n and lambda^n for the old state
            split_b(sB0, u0, dir > 0 ? (lastf ? (r < nrow ? pw[nrow - 1 - r] : 0.f) : pw[255 - r]) : pw[128 + r]);
            sync_tmem();
            if (tid == 0) {
                mma_dw(tD, sB0, sC0, 0, 8, true);
                mma_commit(barM);
            }
            wait_m(86);
            if (!ok) break;
            split_b(sB1, u1,
                    dir > 0 ? (lastf ? (128 + r < nrow ? pw[nrow - 1 - 128 - r] : 0.f) : pw[127 - r]) : pw[r]);
            sync_tmem();
            if (tid == 0) {
                mma_dw(tD, sB1, sC1, 0, 8, false);
                mma_commit(barM);
            }
            wait_m(87);
            if (!ok) break;
            update_w(tD, lastf ? pw[nrow] : (firstr ? pw[nrow - 1] : pw[256]), sW);
            sync_tmem();
        }
    } else {
        const uint32_t tS = tmem, tX = tmem + 128, tY1 = tmem + 192, tY2 = tmem + 256, tD = tmem + 320;
        const int nlast = T - 128 * (nb - 1);  // rows of the last 128-row tile
        for (int step = 0; step < nb && ok; ++step) {
            const int tile = dir > 0 ? step : nb - 1 - step;
            // the two 64-row blocks in scan order: f first, then s (time
            // blocks 0 = rows 0..63, 1 = rows 64..127)
            const int bf = dir > 0 ? 0 : 1;
            // rows of f and s that hold positions of the sequence: all 64,
            // except in the forward scan's last tile (the state after position
            // T-1) and the reverse scan's first tile (the state entering at T-1)
            const bool lastf = dir > 0 && step == nb - 1;
            const bool firstr = dir < 0 && step == 0;
            int nf = 64, nsb = 64;
            if (lastf) {
                nf = min(nlast, 64);
                nsb = max(nlast - 64, 0);
            } else if (firstr) {
                nf = max(nlast - 64, 0);
                nsb = min(nlast, 64);
            }
            if (tid == 0) {
                mbar_arrive_expect_tx(barT, 2 * L::kAsz + L::kCsz);
                load_tile(sB, &R.tb, tile, DA, 0);
                load_tile(sC, &R.tc, tile, kDC, kDC * cs);
                load_tile(sA, &R.ta, tile, DA, 0);
                // the next tile's B, C and A
                const int nt = dir > 0 ? tile + 1 : tile - 1;
                prefetch_tile(&R.tb, nt, DA, 0);
                prefetch_tile(&R.tc, nt, kDC, kDC * cs);
                prefetch_tile(&R.ta, nt, DA, 0);
            }
            wait_t(91);
            if (tid == 0) {
                mma_s(tS, sB);
                mma_xw(tY1, sW);
                mma_commit(barM);
            }
            wait_m(92);
            if (!ok) break;
            // P: the two 64 x 64 diagonal blocks only; w_s B with each block's
            // own weights (lambda^(63-c') forward, lambda^c' reverse)
            auto diag64 = [&](int rr, int c) -> float {
                if ((rr >> 6) != (c >> 6)) return 0.f;
                return dir > 0 ? (c <= rr ? pw[rr - c] : 0.f) : (c >= rr ? pw[c - rr] : 0.f);
            };
            make_p(tS, tile, diag64);
            // forward key weights lambda^(n-1-r') over the block's n rows (n = 64
            // but in the last tile); reverse lambda^r'
            const int nkb = ((r >> 6) == bf) ? nf : nsb;
            split_b(sB, tile, dir > 0 ? ((r & 63) < nkb ? pw[nkb - 1 - (r & 63)] : 0.f) : pw[r & 63]);
            sync_tmem();
            if (tid == 0) {
                mma_pc(tX, tS, sC, true);
                mma_dw(tD, sB, sC, 4 * bf, 4 * bf + 4, true);
                mma_commit(barM);
            }
            wait_m(93);
            if (!ok) break;
            // W_mid, the state after block f: lambda^n_f W + dW_f forward; in
            // the reverse scan's first tile the entering state decays from
            // position T-1 to the start of f (lambda^(n_f-1)), or passes to s
            // unchanged when f holds no position
            update_w(tD, dir > 0 ? pw[nf] : (firstr ? pw[max(nf - 1, 0)] : pw[64]), sW2);
            sync_tmem();
            if (tid == 0) {
                mma_xw(tY2, sW2);
                mma_dw(tD, sB, sC, 4 * (1 - bf), 4 * (1 - bf) + 4, true);
                mma_commit(barM);
            }
            wait_m(94);
            if (!ok) break;
            // rows of f read W, rows of s W_mid, each with its block-local
            // weight lambda^(r'+1) (fwd) or lambda^(64-r') (rev)
            const int rb = r & 63;
            const bool in_f = (r >> 6) == bf;
            float wx = dir > 0 ? pw[rb + 1] : pw[64 - rb];
            if (firstr) {  // the entering state: lambda^(n-1-r') over the n rows that hold it
                if (in_f) wx = rb < nf ? pw[nf - 1 - rb] : 0.f;
                else if (nf == 0) wx = rb < nsb ? pw[nsb - 1 - rb] : 0.f;
            }
            store_x(tX, in_f ? tY1 : tY2, wx, tile);
            // W after block s
            update_w(tD, dir > 0 ? pw[nsb] : ((firstr && nf == 0) ? pw[max(nsb - 1, 0)] : pw[64]), sW);
            sync_tmem();
        }
    }

    // the final state: forward, the state after position T-1; reverse, lambda
    // times the state at position 0
    if (ok && R.fin != nullptr && owns_w_row) {
        float* fin = R.fin + static_cast<size_t>(bh) * (DA * p.dc) + static_cast<size_t>(wrow) * p.dc + kDC * cs +
                     32 * hf;
        const float fs = dir > 0 ? 1.f : lam;
#pragma unroll
        for (int u = 0; u < 32; ++u) fin[u] = fs * wreg[u];
    }

    // tear-down
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace blk
}  // namespace la2
