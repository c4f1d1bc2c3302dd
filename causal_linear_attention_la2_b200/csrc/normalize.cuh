// normalize.cuh -- the normalised form of causal linear attention.
//
// The "Lightning Attention" explainer (section 1) writes causal linear
// attention with a denominator, phi(q_t)^T sum_{s<=t} phi(k_s) v_s^T divided
// by phi(q_t)^T sum_{s<=t} phi(k_s), and says (section 2) that the
// denominator's running sum z is a parallel recurrence next to the state.  With
// the identity feature map (its default; another phi is applied to q and k by
// the caller) and the per-head decay on both sums:
//
//   z_t = lambda z_{t-1} + k_t,   den_t = q_t . z_t,   y_t = num_t / den_t,
//
// num being the unnormalised output of la2_fwd.  Its backward, for dy:
//
//   dnum_t = dy_t / den_t,   dden_t = -(dy_t . y_t) / den_t,
//   dq_t  += dden_t z_t,      dk_s  += sum_{t>=s} lambda^(t-s) dden_t q_t,
//
// with dq, dk, dv of the numerator from la2_bwd given dnum as dout.
//
// Each of these sums over positions is a decayed scan of d-vectors, x_t =
// lambda x_{t-1} + w_t a_t (forward) or x_t = lambda x_{t+1} + w_t a_t
// (reverse): one thread per feature walks the rows of a chunk, which is cheap
// next to the d x e scans, so it is SIMT and bound by memory.  A sequence is cut
// into chunks so that the GPU fills; a pre-pass gives each chunk its incoming x
// (Horner's rule over the end states of the chunks before it in scan order).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace la2 {

constexpr int kNzThreads = 128;  // one per feature (d <= 128)
constexpr int kNzRows = 16;      // rows whose loads are issued together (registers bound occupancy)

enum NzMode { kNzDen = 0, kNzDq = 1, kNzDk = 2 };

struct NzParams {
    const void* a;          // the scanned rows [B, H, T, d] (k: den and dq modes; q: dk mode)
    const void* q;          // den mode: q, dotted with x
    float* y;               // den mode: the numerator, divided in place by den (or null)
    float* den;             // den mode: den [B*H, T] written (or null)
    const float* w;         // dq mode: row factors dden [B*H, T]; dk mode: scan weights dden
    const float* rs;        // dq mode: out_t is first multiplied by rs_t (1 / den_t) [B*H, T]
    float* out;             // dq / dk mode: fp32 [B, H, T, d] (layout of the inputs), added to
    const float* decay;     // [H]
    float* chunk;           // [B*H, nchunk - 1, d]: x at the end of each chunk but the last
    int B, H, T, d, e, bthd;
    int mode, dir;          // NzMode; +1 forward, -1 reverse
    int nchunk, chunk_rows; // chunks per sequence (in scan order) and rows per chunk
};

__device__ __forceinline__ float nz_load(const float* p) { return *p; }
__device__ __forceinline__ float nz_load(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// Rows of sequence bh: row(t) = base + t * stride ([B, H, T, D]: bh T + t;
// [B, T, H, D]: (b T + t) H + h), worked out once per CTA.
struct NzRows {
    size_t base, stride;
    __device__ __forceinline__ NzRows(const NzParams& p, int bh) {
        const int b = bh / p.H, h = bh - b * p.H;
        base = p.bthd ? static_cast<size_t>(b) * p.T * p.H + h : static_cast<size_t>(bh) * p.T;
        stride = p.bthd ? static_cast<size_t>(p.H) : 1;
    }
    __device__ __forceinline__ size_t operator()(int t) const { return base + static_cast<size_t>(t) * stride; }
};

// Rows of chunk j (scan order): [lo, hi) in time.
__device__ __forceinline__ void nz_span(const NzParams& p, int j, int& lo, int& hi) {
    const int c = p.dir > 0 ? j : p.nchunk - 1 - j;
    lo = c * p.chunk_rows;
    hi = min(p.T, lo + p.chunk_rows);
}

// The scan weight of row t: dden_t in dk mode, else 1.
__device__ __forceinline__ float nz_weight(const NzParams& p, int bh, int t) {
    return p.mode == kNzDk ? p.w[static_cast<size_t>(bh) * p.T + t] : 1.f;
}

// Pre-pass: x at the end of chunk j < nchunk - 1 (scan order), from zero.
template <typename Tin>
__global__ void __launch_bounds__(kNzThreads) la2_nz_prepass(const __grid_constant__ NzParams p) {
    const int bh = blockIdx.x / (p.nchunk - 1), j = blockIdx.x % (p.nchunk - 1);
    const int i = threadIdx.x;
    const float lam = p.decay[bh % p.H];
    int lo, hi;
    nz_span(p, j, lo, hi);
    const Tin* a = static_cast<const Tin*>(p.a);
    const NzRows nz_row(p, bh);
    float x = 0.f;
    const int n = hi - lo;
    const int ic = min(i, p.d - 1);
    for (int s0 = 0; s0 < n; s0 += kNzRows) {
        const int m = min(kNzRows, n - s0);
        // every load of the batch first (addresses clamped into range, so that
        // none waits behind a branch), then the recurrence
        float av[kNzRows], wv[kNzRows];
#pragma unroll
        for (int r = 0; r < kNzRows; ++r) {
            const int rr = min(r, m - 1);
            const int t = p.dir > 0 ? lo + s0 + rr : hi - 1 - s0 - rr;
            av[r] = nz_load(a + nz_row(t) * p.d + ic);
            wv[r] = nz_weight(p, bh, t);
        }
#pragma unroll
        for (int r = 0; r < kNzRows; ++r)
            if (r < m) x = fmaf(lam, x, wv[r] * av[r]);
    }
    if (i < p.d) p.chunk[(static_cast<size_t>(bh) * (p.nchunk - 1) + j) * p.d + i] = x;
}

// Main pass over chunk j (scan order) of each sequence.
template <typename Tin>
__global__ void __launch_bounds__(kNzThreads) la2_nz_scan(const __grid_constant__ NzParams p) {
    __shared__ float part[kNzThreads / 32][kNzRows];
    __shared__ float dens[kNzRows];
    const int bh = blockIdx.x / p.nchunk, j = blockIdx.x % p.nchunk;
    const int i = threadIdx.x, warp = i >> 5, lane = i & 31;
    const double l2 = log2(static_cast<double>(p.decay[bh % p.H]));
    const float lam = p.decay[bh % p.H];
    int lo, hi;
    nz_span(p, j, lo, hi);
    // incoming x: Horner's rule over the end states of chunks 0 .. j-1
    float x = 0.f;
    for (int g = 0; g < j; ++g) {
        int glo, ghi;
        nz_span(p, g, glo, ghi);
        const float f = static_cast<float>(exp2(static_cast<double>(ghi - glo) * l2));
        const float xe = i < p.d ? p.chunk[(static_cast<size_t>(bh) * (p.nchunk - 1) + g) * p.d + i] : 0.f;
        x = fmaf(f, x, xe);
    }
    const Tin* a = static_cast<const Tin*>(p.a);
    const Tin* q = static_cast<const Tin*>(p.q);
    const NzRows nz_row(p, bh);
    const int n = hi - lo;
    const int ic = min(i, p.d - 1);
    const float fi = i < p.d ? 1.f : 0.f;  // threads past d carry zeros
    for (int s0 = 0; s0 < n; s0 += kNzRows) {
        const int m = min(kNzRows, n - s0);
        // every load of the batch first, addresses clamped into range (rows
        // past m repeat the last row and are not used), then the recurrence
        float av[kNzRows], wv[kNzRows], qv[kNzRows];
#pragma unroll
        for (int r = 0; r < kNzRows; ++r) {
            const int rr = min(r, m - 1);
            const int t = p.dir > 0 ? lo + s0 + rr : hi - 1 - s0 - rr;
            const size_t row = nz_row(t);
            av[r] = fi * nz_load(a + row * p.d + ic);
            wv[r] = r < m ? nz_weight(p, bh, t) : 0.f;
            if (p.mode == kNzDen) qv[r] = nz_load(q + row * p.d + ic);
            else qv[r] = p.out[row * p.d + ic];       // dq / dk mode: the row to add to
        }
        if (p.mode == kNzDen) {
            // den_t = q_t . x_t: per row a warp sum, then the four warps' sums
#pragma unroll
            for (int r = 0; r < kNzRows; ++r) {
                x = fmaf(lam, x, wv[r] * av[r]);
                float pr = qv[r] * x;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) pr += __shfl_xor_sync(0xffffffffu, pr, o);
                if (lane == 0) part[warp][r] = pr;
            }
            __syncthreads();
            if (i < kNzRows && i < m) {
                float s = 0.f;
#pragma unroll
                for (int w = 0; w < kNzThreads / 32; ++w) s += part[w][i];
                dens[i] = s;
                if (p.den) p.den[static_cast<size_t>(bh) * p.T + lo + s0 + i] = s;
            }
            __syncthreads();
            if (p.y) {
                // y rows of the batch: all loads, then the divisions and stores
                constexpr int kPer = kNzRows * 128 / kNzThreads;  // e <= 128
                float yv[kPer];
#pragma unroll
                for (int u = 0; u < kPer; ++u) {
                    const int z = i + u * kNzThreads, r = z >> 7, c = z & 127;
                    yv[u] = (r < m && c < p.e) ? p.y[nz_row(lo + s0 + r) * p.e + c] : 0.f;
                }
#pragma unroll
                for (int u = 0; u < kPer; ++u) {
                    const int z = i + u * kNzThreads, r = z >> 7, c = z & 127;
                    if (r < m && c < p.e) p.y[nz_row(lo + s0 + r) * p.e + c] = yv[u] / dens[r];
                }
            }
            __syncthreads();
        } else {
            // dq: out_t = rs_t out_t + dden_t x_t (forward scan of k); dk:
            // out_t += x_t (reverse scan of dden_t q_t); the rows of out were
            // read with the batch's loads (qv), so no load waits behind a store
            float fv[kNzRows], sv[kNzRows];
#pragma unroll
            for (int r = 0; r < kNzRows; ++r) {
                const int rr = min(r, m - 1);
                const size_t st = static_cast<size_t>(bh) * p.T + (p.dir > 0 ? lo + s0 + rr : hi - 1 - s0 - rr);
                fv[r] = p.mode == kNzDq ? p.w[st] : 1.f;
                sv[r] = p.mode == kNzDq ? p.rs[st] : 1.f;
            }
#pragma unroll
            for (int r = 0; r < kNzRows; ++r) {
                x = fmaf(lam, x, wv[r] * av[r]);
                qv[r] = fmaf(fv[r], x, qv[r] * sv[r]);
            }
            if (i < p.d) {
#pragma unroll
                for (int r = 0; r < kNzRows; ++r) {
                    if (r < m) {
                        const int t = p.dir > 0 ? lo + s0 + r : hi - 1 - s0 - r;
                        p.out[nz_row(t) * p.d + i] = qv[r];
                    }
                }
            }
        }
    }
}

// The backward's first step, one warp per row (sequence bh, position t):
// dden_t = -(dy_t . y_t) / den_t and inv_t = 1 / den_t, the factor with which
// dnum_t = dy_t / den_t enters the backward scans (in fp32, inside them).
template <typename Tin>
__global__ void la2_nz_prep(const Tin* dy, const float* y, const float* den, float* dden, float* inv,
                            long long rows, int H, int T, int e, int bthd) {
    const long long wid = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (wid >= rows) return;
    const long long bh = wid / T;
    const int t = static_cast<int>(wid - bh * T);
    const long long b = bh / H, h = bh - b * H;
    const size_t row = bthd ? static_cast<size_t>((b * T + t) * H + h) : static_cast<size_t>(wid);
    const float dn = den[wid];
    float s = 0.f;
    for (int c = lane; c < e; c += 32) s = fmaf(nz_load(dy + row * e + c), y[row * e + c], s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) {
        dden[wid] = -s / dn;
        inv[wid] = 1.f / dn;
    }
}

}  // namespace la2
