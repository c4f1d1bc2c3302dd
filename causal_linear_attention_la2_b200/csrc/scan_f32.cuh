// scan_f32.cuh -- fp32 SIMT kernel of the Lightning Attention-2 path.
//
// Same decayed scan as the tcgen05 kernel (see scan_ws_sm100.cuh), in plain
// fp32 FFMA so that fp32 inputs keep fp32 accuracy (tensor cores would round
// operands to bf16/tf32).  The tile length T_B (64, 128 or 256) is honoured:
// the state W is carried from tile to tile and updated once per tile; inside a
// tile the intra-tile product is formed 64 rows by 64 columns at a time to
// bound shared memory.  One CTA per (sequence, role); any DA, DC <= 128.
#pragma once
#include <cstdint>

namespace la2 {

constexpr int kF32Threads = 256;
constexpr int kF32Sub = 64;

struct F32Role {
    const float* a;  // [BH, T, DA]
    const float* b;  // [BH, T, DA]
    const float* c;  // [BH, T, DC]
    float* x;        // [BH, T, DC]
    const float* init;  // [BH, DA, DC] state the scan starts from, or null (0); with
                        // init_t, [BH, DC, DA] read transposed
    float* fin;         // [BH, DA, DC] state the scan ends with, or null
    int da, dc, dir;
    int init_t;
    const float* colf;  // [BH, T] factor on the summed position, or null (see scan_ws_sm100.cuh)
    // dir = +1: init is the state before position 0, fin the state after
    // position T-1.  dir = -1: init enters at position T-1 (row t weighs it by
    // lambda^(T-1-t)), and fin is lambda times the state at position 0.
};

struct F32Params {
    F32Role role[3];
    const float* decay;
    int H, T, TB, nroles;
    int bthd;  // 0: [B, H, T, D]; 1: [B, T, H, D]
};

__host__ __device__ inline size_t f32_scan_smem_bytes(int da, int dc, int TB) {
    return sizeof(float) * (static_cast<size_t>(da) * dc + 2 * kF32Sub * da + kF32Sub * dc +
                            kF32Sub * kF32Sub + (TB + 1));
}

__global__ void __launch_bounds__(kF32Threads)
la2_scan_f32(const __grid_constant__ F32Params p)
{
    extern __shared__ float fsm[];
    const int role_id = blockIdx.x % p.nroles;
    const int bh = blockIdx.x / p.nroles;
    const F32Role R = p.role[role_id];
    const int da = R.da, dc = R.dc, dir = R.dir, T = p.T, TB = p.TB;

    float* W = fsm;                               // [da][dc]
    float* As = W + da * dc;                      // [64][da]
    float* Bs = As + kF32Sub * da;                // [64][da]
    float* Cs = Bs + kF32Sub * da;                // [64][dc]
    float* Ps = Cs + kF32Sub * dc;                // [64][64]
    float* pw = Ps + kF32Sub * kF32Sub;           // lambda^n, n = 0..TB

    const int tid = threadIdx.x;
    const double lam = static_cast<double>(p.decay[bh % p.H]);
    const double l2 = log2(lam);
    for (int n = tid; n <= TB; n += kF32Threads) pw[n] = static_cast<float>(exp2(n * l2));
    for (int z = tid; z < da * dc; z += kF32Threads) {
        const int u = z / dc, j = z % dc;
        W[z] = R.init ? R.init[static_cast<size_t>(bh) * da * dc +
                               (R.init_t ? static_cast<size_t>(j) * da + u : static_cast<size_t>(z))]
                      : 0.f;
    }

    // sequence bh: base row and row stride in units of D ([B,H,T,D]: bh T, 1;
    // [B,T,H,D]: b T H + h, H)
    const size_t rs = p.bthd ? static_cast<size_t>(p.H) : 1;
    const size_t r0 = p.bthd ? static_cast<size_t>(bh / p.H) * T * p.H + bh % p.H
                             : static_cast<size_t>(bh) * T;
    const float* a = R.a + r0 * da;
    const float* b = R.b + r0 * da;
    const float* c = R.c + r0 * dc;
    float* x = R.x + r0 * dc;

    const int nb = (T + TB - 1) / TB;
    const int row = tid >> 2;   // 0..63: row of the 64-row sub-tile this thread accumulates
    const int jc = tid & 3;     // columns jc, jc+4, ...
    __syncthreads();

    for (int step = 0; step < nb; ++step) {
        const int i = dir > 0 ? step : nb - 1 - step;
        const int t0 = i * TB;
        const int len = min(TB, T - t0);
        const int nsub = (len + kF32Sub - 1) / kF32Sub;

        for (int qa = 0; qa < nsub; ++qa) {
            // query sub-tile
            for (int z = tid; z < kF32Sub * da; z += kF32Threads) {
                const int rr = z / da, u = z % da, loc = qa * kF32Sub + rr;
                As[z] = loc < len ? a[static_cast<size_t>(t0 + loc) * rs * da + u] : 0.f;
            }
            __syncthreads();

            // inter-tile term: w_x(r) * a_r^T W
            float acc[32];
            const int rloc = qa * kF32Sub + row;
            // the reverse scan's first tile (the sequence's last) takes the
            // entering state at position T-1: lambda^(len-1-r)
            const float wx = dir > 0 ? pw[min(rloc + 1, TB)]
                                     : (step == 0 ? pw[max(len - 1 - rloc, 0)] : pw[max(TB - rloc, 0)]);
#pragma unroll
            for (int m = 0; m < 32; ++m) {
                const int j = jc + 4 * m;
                float s = 0.f;
                if (j < dc)
                    for (int u = 0; u < da; ++u) s = fmaf(As[row * da + u], W[u * dc + j], s);
                acc[m] = wx * s;
            }

            // intra-tile term over the key sub-tiles on the causal side
            for (int kb = 0; kb < nsub; ++kb) {
                if (dir > 0 ? kb > qa : kb < qa) continue;
                __syncthreads();
                for (int z = tid; z < kF32Sub * da; z += kF32Threads) {
                    const int rr = z / da, u = z % da, loc = kb * kF32Sub + rr;
                    Bs[z] = loc < len ? b[static_cast<size_t>(t0 + loc) * rs * da + u] : 0.f;
                }
                for (int z = tid; z < kF32Sub * dc; z += kF32Threads) {
                    const int rr = z / dc, j = z % dc, loc = kb * kF32Sub + rr;
                    Cs[z] = loc < len ? c[static_cast<size_t>(t0 + loc) * rs * dc + j] : 0.f;
                }
                __syncthreads();
                for (int z = tid; z < kF32Sub * kF32Sub; z += kF32Threads) {
                    const int rr = z / kF32Sub, cc = z % kF32Sub;
                    const int lag = dir > 0 ? (qa * kF32Sub + rr) - (kb * kF32Sub + cc)
                                            : (kb * kF32Sub + cc) - (qa * kF32Sub + rr);
                    float s = 0.f;
                    if (lag >= 0) {
                        for (int u = 0; u < da; ++u) s = fmaf(As[rr * da + u], Bs[cc * da + u], s);
                        s *= pw[lag];
                        const int loc = kb * kF32Sub + cc;
                        if (R.colf) s *= loc < len ? R.colf[static_cast<size_t>(bh) * T + t0 + loc] : 0.f;
                    }
                    Ps[z] = s;
                }
                __syncthreads();
#pragma unroll
                for (int m = 0; m < 32; ++m) {
                    const int j = jc + 4 * m;
                    if (j < dc) {
                        float s = acc[m];
                        for (int cc = 0; cc < kF32Sub; ++cc)
                            s = fmaf(Ps[row * kF32Sub + cc], Cs[cc * dc + j], s);
                        acc[m] = s;
                    }
                }
            }
            if (rloc < len) {
#pragma unroll
                for (int m = 0; m < 32; ++m) {
                    const int j = jc + 4 * m;
                    if (j < dc) x[static_cast<size_t>(t0 + rloc) * rs * dc + j] = acc[m];
                }
            }
            __syncthreads();
        }

        // state update with the unmasked tile: W <- lambda^TB W + sum_c w_s(c) b_c c_c^T.
        // A forward scan's last tile may be short (len < TB rows): its exponents
        // are taken from len, so that W is then the state after position T-1
        // (no output reads it; the final state does).
        // A reverse scan's first tile decays the entering state by lambda^(len-1).
        const int tl = dir > 0 ? len : TB;
        const float lTB = (dir < 0 && step == 0) ? pw[len - 1] : pw[tl];
        for (int z = tid; z < da * dc; z += kF32Threads) W[z] *= lTB;
        for (int kb = 0; kb < nsub; ++kb) {
            __syncthreads();
            for (int z = tid; z < kF32Sub * da; z += kF32Threads) {
                const int rr = z / da, u = z % da, loc = kb * kF32Sub + rr;
                float ws = loc < len ? (dir > 0 ? pw[tl - 1 - loc] : pw[loc]) : 0.f;
                if (R.colf && loc < len) ws *= R.colf[static_cast<size_t>(bh) * T + t0 + loc];
                Bs[z] = loc < len ? ws * b[static_cast<size_t>(t0 + loc) * rs * da + u] : 0.f;
            }
            for (int z = tid; z < kF32Sub * dc; z += kF32Threads) {
                const int rr = z / dc, j = z % dc, loc = kb * kF32Sub + rr;
                Cs[z] = loc < len ? c[static_cast<size_t>(t0 + loc) * rs * dc + j] : 0.f;
            }
            __syncthreads();
            for (int z = tid; z < da * dc; z += kF32Threads) {
                const int u = z / dc, j = z % dc;
                float s = W[z];
                for (int cc = 0; cc < kF32Sub; ++cc) s = fmaf(Bs[cc * da + u], Cs[cc * dc + j], s);
                W[z] = s;
            }
        }
        __syncthreads();
    }
    if (R.fin) {
        const float fs = dir > 0 ? 1.f : static_cast<float>(lam);
        for (int z = tid; z < da * dc; z += kF32Threads)
            R.fin[static_cast<size_t>(bh) * da * dc + z] = fs * W[z];
    }
}

}  // namespace la2
