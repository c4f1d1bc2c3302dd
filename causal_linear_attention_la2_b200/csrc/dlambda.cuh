// dlambda.cuh -- gradient of the loss with respect to the per-head decay.
//
// For the forward from S_{-1} = S0 (S_t = lambda S_{t-1} + k_t v_t^T,
// o_t = S_t^T q_t) and L = sum_t dout_t . o_t + <G, S_{T-1}>, the derivative
// U_t = dS_t/dlambda obeys U_t = lambda U_{t-1} + S_{t-1} (U_{-1} = 0), and
//
//     dL/dlambda = sum_t q_t^T U_t dout_t + <G, U_{T-1}>,
//
// i.e. the lag-weighted form sum_{s<t} (t-s) lambda^(t-s-1) (q_t.k_s)(do_t.v_s)
// plus the terms of S0 and G.  It is the decay of the "Lightning Attention"
// explainer's recurrence (section 1) differentiated; the tiling follows its
// section 2: inside a sub-tile of n <= 32 rows (local row r, column c, states
// W = S and U at the position before the sub-tile)
//
//   inter  sum_r (r+1) lambda^r q_r^T W do_r + lambda^(r+1) q_r^T U do_r
//   intra  sum_{r>c} (r-c) lambda^(r-c-1) (q_r . k_c)(do_r . v_c)
//   carry  W <- lambda^n W + sum_c lambda^(n-1-c) k_c v_c^T
//          U <- n lambda^(n-1) W + lambda^n U + sum_c (n-1-c) lambda^(n-2-c) k_c v_c^T
//
// The result is one scalar per head, so these kernels are SIMT fp32 (fp64
// accumulation of the scalar): 256 threads per CTA, each owning an 8 x 8 block
// of W and U in registers (rows {4a+i, 64+4a+i}, columns likewise, so that the
// float4 reads of a quarter-warp cover 128 contiguous bytes).  A sequence is cut
// into up to 32 segments so that few sequences still fill the GPU; a pre-pass
// computes each segment's end states (W, U) from zero, and each segment then
// starts from the states its predecessors leave (Horner's rule over them).
// Partial sums go to the workspace and a last launch adds them per head in a
// fixed order, so the result is deterministic.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace la2 {

constexpr int kDlThreads = 256;
constexpr int kDlRows = 32;       // rows of a sub-tile
constexpr int kDlStride = 132;    // floats per smem row (16-byte aligned, conflict-free float4)

struct DlParams {
    const void* q;
    const void* k;
    const void* v;
    const void* g;          // dout
    const float* decay;     // [H]
    const float* init;      // [BH, d, e] S0, or null
    const float* dfin;      // [BH, d, e] G, or null
    float* seg_state;       // [BH, nseg - 1, 2, d, e]: (W, U) at the end of each segment but the last
    double* partial;        // [BH, nseg]
    float* d_decay;         // [H]
    int B, H, T, d, e, bthd;
    int nseg, seg_rows;     // segments per sequence and rows per segment (a multiple of kDlRows)
    int vec;                // 1: d and e are multiples of 16 bytes of elements (vector staging)
};

__device__ __forceinline__ float dl_load(const float* p) { return *p; }
__device__ __forceinline__ float dl_load(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// Rows of sequence bh: row(t) = base + t * stride ([B, H, T, D]: bh T + t;
// [B, T, H, D]: (b T + t) H + h), worked out once per CTA.
struct DlRows {
    size_t base, stride;
    __device__ __forceinline__ DlRows(const DlParams& p, int bh) {
        const int b = bh / p.H, h = bh - b * p.H;
        base = p.bthd ? static_cast<size_t>(b) * p.T * p.H + h : static_cast<size_t>(bh) * p.T;
        stride = p.bthd ? static_cast<size_t>(p.H) : 1;
    }
    __device__ __forceinline__ size_t operator()(int t) const { return base + static_cast<size_t>(t) * stride; }
};

__device__ __forceinline__ void dl_cvt(uint4 w, const float*, float (&x)[4]) {
    x[0] = __uint_as_float(w.x); x[1] = __uint_as_float(w.y);
    x[2] = __uint_as_float(w.z); x[3] = __uint_as_float(w.w);
}
__device__ __forceinline__ void dl_cvt(uint4 w, const __nv_bfloat16*, float (&x)[8]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(u[i] << 16);
        x[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
}

// Rows [t0, t0 + n) of sequence bh of two [B, H, T, D] (or [B, T, H, D])
// tensors into smem as fp32 rows of kDlStride floats, zero past n rows and D
// columns.  With p.vec (every D a multiple of 16 bytes of elements) each
// thread reads 16-byte vectors, all of both tensors' loads issued before any
// store; otherwise element by element, loads again batched ahead of stores.
template <typename Tin>
__device__ __forceinline__ void dl_stage2(float* dA, const Tin* sA, int DA, float* dB, const Tin* sB, int DB,
                                          const DlParams& p, const DlRows& dl_row, int t0, int n) {
    if (p.vec) {
        constexpr int kE = 16 / sizeof(Tin);                   // elements per vector
        constexpr int kCh = 128 / kE;                          // vectors per smem row
        constexpr int kPer = kDlRows * kCh / kDlThreads;       // vectors per thread and tensor
        uint4 va[kPer], vb[kPer];
#pragma unroll
        for (int m = 0; m < kPer; ++m) {
            const int z = threadIdx.x + m * kDlThreads, r = z / kCh, c = (z % kCh) * kE;
            const size_t row = dl_row(t0 + r);
            va[m] = (r < n && c < DA) ? __ldg(reinterpret_cast<const uint4*>(sA + row * DA + c)) : make_uint4(0, 0, 0, 0);
            vb[m] = (r < n && c < DB) ? __ldg(reinterpret_cast<const uint4*>(sB + row * DB + c)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int m = 0; m < kPer; ++m) {
            const int z = threadIdx.x + m * kDlThreads, r = z / kCh, c = (z % kCh) * kE;
            float x[kE], y[kE];
            dl_cvt(va[m], sA, x);
            dl_cvt(vb[m], sB, y);
#pragma unroll
            for (int i = 0; i < kE; i += 4) {
                *reinterpret_cast<float4*>(dA + r * kDlStride + c + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
                *reinterpret_cast<float4*>(dB + r * kDlStride + c + i) = make_float4(y[i], y[i + 1], y[i + 2], y[i + 3]);
            }
        }
        return;
    }
    constexpr int kPer = kDlRows * 128 / kDlThreads;  // 16 elements per thread and tensor
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        float* dst = half ? dB : dA;
        const Tin* src = half ? sB : sA;
        const int D = half ? DB : DA;
        float x[kPer];
#pragma unroll
        for (int m = 0; m < kPer; ++m) {
            const int z = threadIdx.x + m * kDlThreads, r = z >> 7, u = z & 127;
            x[m] = (r < n && u < D) ? dl_load(src + dl_row(t0 + r) * D + u) : 0.f;
        }
#pragma unroll
        for (int m = 0; m < kPer; ++m) {
            const int z = threadIdx.x + m * kDlThreads, r = z >> 7, u = z & 127;
            dst[r * kDlStride + u] = x[m];
        }
    }
}

// L2 prefetch of rows [t0, t0 + n) of sequence bh of a tensor (one 128-byte
// line per thread and call at most), so that the next staging reads L2.
template <typename Tin>
__device__ __forceinline__ void dl_prefetch(const Tin* src, int D, const DlRows& dl_row, int t0, int n) {
    const int lines = (D * static_cast<int>(sizeof(Tin)) + 127) / 128;
    const int z = threadIdx.x;
    if (z < n * lines) {
        const int r = z / lines, l = z % lines;
        const char* a = reinterpret_cast<const char*>(src + dl_row(t0 + r) * D) + 128 * l;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
    }
}

// Columns (or rows) of the state block a thread owns: {4a + i, 64 + 4a + i}.
__device__ __forceinline__ int dl_idx(int a, int m) { return (m < 4 ? 4 * a + m : 64 + 4 * a + (m - 4)); }

__device__ __forceinline__ void dl_ld8(const float* row, int a, float (&x)[8]) {
    const float4 lo = *reinterpret_cast<const float4*>(row + 4 * a);
    const float4 hi = *reinterpret_cast<const float4*>(row + 64 + 4 * a);
    x[0] = lo.x; x[1] = lo.y; x[2] = lo.z; x[3] = lo.w;
    x[4] = hi.x; x[5] = hi.y; x[6] = hi.z; x[7] = hi.w;
}

// lambda^m as float, m >= 0 (lambda^0 = 1)
__device__ __forceinline__ float dl_pow(double l2, double m) {
    return m == 0.0 ? 1.f : static_cast<float>(exp2(m * l2));
}

// pw[m] = lambda^m, m = 0 .. kDlRows (every exponent inside a sub-tile)
__device__ __forceinline__ void dl_table(float* pw, double l2) {
    for (int m = threadIdx.x; m <= kDlRows; m += kDlThreads) pw[m] = dl_pow(l2, m);
}

// The carry over one sub-tile of n rows (Ks, Vs staged): W, U <- as in the
// header, for this thread's 8 x 8 block.
__device__ __forceinline__ void dl_carry(float (&W)[64], float (&U)[64], const float* Ks, const float* Vs,
                                         int n, const float* pw, int ti, int tj) {
    const float ln = pw[n], nln1 = static_cast<float>(n) * pw[n - 1];
#pragma unroll
    for (int z = 0; z < 64; ++z) {
        U[z] = fmaf(nln1, W[z], ln * U[z]);
        W[z] *= ln;
    }
    for (int c = 0; c < n; ++c) {
        const float ws = pw[n - 1 - c];
        const float wu = (n - 1 - c) > 0 ? static_cast<float>(n - 1 - c) * pw[n - 2 - c] : 0.f;
        float kk[8], vv[8];
        dl_ld8(Ks + c * kDlStride, ti, kk);
        dl_ld8(Vs + c * kDlStride, tj, vv);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float kw = ws * kk[i], ku = wu * kk[i];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                W[i * 8 + j] = fmaf(kw, vv[j], W[i * 8 + j]);
                U[i * 8 + j] = fmaf(ku, vv[j], U[i * 8 + j]);
            }
        }
    }
}

// Pre-pass: (W, U) at the end of segment j < nseg - 1 of each sequence, from zero.
template <typename Tin>
__global__ void __launch_bounds__(kDlThreads, 1) la2_dlam_prepass(const __grid_constant__ DlParams p) {
    extern __shared__ __align__(16) float dsm[];
    float* Ks = dsm;
    float* Vs = Ks + kDlRows * kDlStride;
    float* pw = Vs + kDlRows * kDlStride;
    const int bh = blockIdx.x / (p.nseg - 1), j = blockIdx.x % (p.nseg - 1);
    const int tid = threadIdx.x, ti = tid >> 4, tj = tid & 15;
    const DlRows rows(p, bh);
    const double l2 = log2(static_cast<double>(p.decay[bh % p.H]));
    dl_table(pw, l2);
    const int a = j * p.seg_rows, bnd = min(p.T, a + p.seg_rows);
    float W[64], U[64];
#pragma unroll
    for (int z = 0; z < 64; ++z) W[z] = U[z] = 0.f;
    for (int t0 = a; t0 < bnd; t0 += kDlRows) {
        const int n = min(kDlRows, bnd - t0);
        __syncthreads();
        dl_stage2(Ks, static_cast<const Tin*>(p.k), p.d, Vs, static_cast<const Tin*>(p.v), p.e, p, rows, t0, n);
        __syncthreads();
        if (t0 + kDlRows < bnd) {
            const int nn = min(kDlRows, bnd - t0 - kDlRows);
            dl_prefetch(static_cast<const Tin*>(p.k), p.d, rows, t0 + kDlRows, nn);
            dl_prefetch(static_cast<const Tin*>(p.v), p.e, rows, t0 + kDlRows, nn);
        }
        dl_carry(W, U, Ks, Vs, n, pw, ti, tj);
    }
    float* dst = p.seg_state + (static_cast<size_t>(bh) * (p.nseg - 1) + j) * 2 * p.d * p.e;
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            const int r = dl_idx(ti, i), c = dl_idx(tj, jj);
            if (r < p.d && c < p.e) {
                dst[static_cast<size_t>(r) * p.e + c] = W[i * 8 + jj];
                dst[static_cast<size_t>(p.d) * p.e + static_cast<size_t>(r) * p.e + c] = U[i * 8 + jj];
            }
        }
}

// Main pass: the partial dL/dlambda of segment j of each sequence.
template <typename Tin>
__global__ void __launch_bounds__(kDlThreads, 1) la2_dlam_scan(const __grid_constant__ DlParams p) {
    extern __shared__ __align__(16) float dsm[];
    float* Qs = dsm;
    float* Ks = Qs + kDlRows * kDlStride;
    float* Vs = Ks + kDlRows * kDlStride;
    float* Gs = Vs + kDlRows * kDlStride;
    double* red = reinterpret_cast<double*>(Gs + kDlRows * kDlStride);  // [kDlThreads / 32]
    float* pw = reinterpret_cast<float*>(red + kDlThreads / 32);         // [kDlRows + 1]
    const int bh = blockIdx.x / p.nseg, j = blockIdx.x % p.nseg;
    const int tid = threadIdx.x, ti = tid >> 4, tj = tid & 15;
    const DlRows rows(p, bh);
    const double l2 = log2(static_cast<double>(p.decay[bh % p.H]));
    dl_table(pw, l2);
    const size_t de = static_cast<size_t>(p.d) * p.e;

    // incoming states: W = S0 (or 0), U = 0, carried over segments 0 .. j-1
    float W[64], U[64];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            const int r = dl_idx(ti, i), c = dl_idx(tj, jj);
            W[i * 8 + jj] = (p.init && r < p.d && c < p.e) ? p.init[bh * de + static_cast<size_t>(r) * p.e + c] : 0.f;
            U[i * 8 + jj] = 0.f;
        }
    for (int g = 0; g < j; ++g) {
        const int n = min(p.seg_rows, p.T - g * p.seg_rows);
        const float ln = dl_pow(l2, n), nln1 = static_cast<float>(n) * dl_pow(l2, n - 1);
        const float* src = p.seg_state + (static_cast<size_t>(bh) * (p.nseg - 1) + g) * 2 * de;
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int r = dl_idx(ti, i), c = dl_idx(tj, jj);
                const bool ok = r < p.d && c < p.e;
                const float ws = ok ? src[static_cast<size_t>(r) * p.e + c] : 0.f;
                const float us = ok ? src[de + static_cast<size_t>(r) * p.e + c] : 0.f;
                const int z = i * 8 + jj;
                U[z] = fmaf(nln1, W[z], fmaf(ln, U[z], us));
                W[z] = fmaf(ln, W[z], ws);
            }
    }

    double acc = 0.0;
    const int a = j * p.seg_rows, bnd = min(p.T, a + p.seg_rows);
    for (int t0 = a; t0 < bnd; t0 += kDlRows) {
        const int n = min(kDlRows, bnd - t0);
        __syncthreads();
        dl_stage2(Qs, static_cast<const Tin*>(p.q), p.d, Ks, static_cast<const Tin*>(p.k), p.d, p, rows, t0, n);
        dl_stage2(Vs, static_cast<const Tin*>(p.v), p.e, Gs, static_cast<const Tin*>(p.g), p.e, p, rows, t0, n);
        __syncthreads();
        if (t0 + kDlRows < bnd) {
            const int nn = min(kDlRows, bnd - t0 - kDlRows);
            dl_prefetch(static_cast<const Tin*>(p.q), p.d, rows, t0 + kDlRows, nn);
            dl_prefetch(static_cast<const Tin*>(p.k), p.d, rows, t0 + kDlRows, nn);
            dl_prefetch(static_cast<const Tin*>(p.v), p.e, rows, t0 + kDlRows, nn);
            dl_prefetch(static_cast<const Tin*>(p.g), p.e, rows, t0 + kDlRows, nn);
        }
        // inter: (r+1) lambda^r q_r^T W do_r + lambda^(r+1) q_r^T U do_r, this
        // thread's block of W and U
        float part = 0.f;
        for (int r = 0; r < n; ++r) {
            float qq[8], gg[8];
            dl_ld8(Qs + r * kDlStride, ti, qq);
            dl_ld8(Gs + r * kDlStride, tj, gg);
            float sw = 0.f, su = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float tw = 0.f, tu = 0.f;
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    tw = fmaf(W[i * 8 + jj], gg[jj], tw);
                    tu = fmaf(U[i * 8 + jj], gg[jj], tu);
                }
                sw = fmaf(qq[i], tw, sw);
                su = fmaf(qq[i], tu, su);
            }
            part = fmaf(static_cast<float>(r + 1) * pw[r], sw, part);
            part = fmaf(pw[r + 1], su, part);
        }
        acc += part;
        // intra: rows r in {ti, ti + 16}, columns c in {tj, tj + 16}, r > c
        {
            float s[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, dp[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
            for (int u = 0; u < 128; u += 4) {
                float4 qa[2], kb[2], ga[2], vb[2];
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    qa[x] = *reinterpret_cast<const float4*>(Qs + (ti + 16 * x) * kDlStride + u);
                    ga[x] = *reinterpret_cast<const float4*>(Gs + (ti + 16 * x) * kDlStride + u);
                    kb[x] = *reinterpret_cast<const float4*>(Ks + (tj + 16 * x) * kDlStride + u);
                    vb[x] = *reinterpret_cast<const float4*>(Vs + (tj + 16 * x) * kDlStride + u);
                }
#pragma unroll
                for (int x = 0; x < 2; ++x)
#pragma unroll
                    for (int y = 0; y < 2; ++y) {
                        s[x][y] = fmaf(qa[x].x, kb[y].x, fmaf(qa[x].y, kb[y].y,
                                  fmaf(qa[x].z, kb[y].z, fmaf(qa[x].w, kb[y].w, s[x][y]))));
                        dp[x][y] = fmaf(ga[x].x, vb[y].x, fmaf(ga[x].y, vb[y].y,
                                   fmaf(ga[x].z, vb[y].z, fmaf(ga[x].w, vb[y].w, dp[x][y]))));
                    }
            }
            float pi = 0.f;
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
                for (int y = 0; y < 2; ++y) {
                    const int r = ti + 16 * x, c = tj + 16 * y;
                    if (r < n && c < r)
                        pi = fmaf(static_cast<float>(r - c) * pw[r - c - 1], s[x][y] * dp[x][y], pi);
                }
            acc += pi;
        }
        dl_carry(W, U, Ks, Vs, n, pw, ti, tj);
    }
    // the last segment: <G, U_{T-1}>
    if (p.dfin && j == p.nseg - 1) {
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int r = dl_idx(ti, i), c = dl_idx(tj, jj);
                if (r < p.d && c < p.e) part = fmaf(p.dfin[bh * de + static_cast<size_t>(r) * p.e + c], U[i * 8 + jj], part);
            }
        acc += part;
    }
    // CTA sum in a fixed order
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((tid & 31) == 0) red[tid >> 5] = acc;
    __syncthreads();
    if (tid == 0) {
        double s = 0.0;
        for (int w = 0; w < kDlThreads / 32; ++w) s += red[w];
        p.partial[static_cast<size_t>(bh) * p.nseg + j] = s;
    }
}

// d_decay[h] = sum over the batch and the segments of the partial sums, in order.
__global__ void la2_dlam_reduce(const __grid_constant__ DlParams p) {
    for (int h = blockIdx.x * blockDim.x + threadIdx.x; h < p.H; h += gridDim.x * blockDim.x) {
        double s = 0.0;
        for (int b = 0; b < p.B; ++b)
            for (int j = 0; j < p.nseg; ++j) s += p.partial[(static_cast<size_t>(b) * p.H + h) * p.nseg + j];
        p.d_decay[h] = static_cast<float>(s);
    }
}

inline size_t dl_scan_smem_bytes() {
    return 4 * sizeof(float) * kDlRows * kDlStride + sizeof(double) * (kDlThreads / 32) +
           sizeof(float) * (kDlRows + 8);
}
inline size_t dl_prepass_smem_bytes() { return 2 * sizeof(float) * kDlRows * kDlStride + sizeof(float) * (kDlRows + 8); }

}  // namespace la2
