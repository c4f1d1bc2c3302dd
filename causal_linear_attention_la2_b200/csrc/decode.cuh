// decode.cuh -- one recurrent step of causal linear attention with decay for
// one new token per sequence:
//
//   S <- lambda_h S + k v^T        (d x e, fp32, updated in place)
//   o  = S^T q                     (e, fp32)
//
// the recurrence of the "Lightning Attention" explainer (section 1, prefix-sum
// form; section 2, memory footprint: the d x e state is all a sequence
// carries), which is what gives generation its constant cost per token.  The
// step reads and writes the state once, so it is bound by memory bandwidth:
// one CTA per sequence, 256 threads; a warp reads whole rows of the state
// (float4 per thread, e % 4 == 0) or single floats (otherwise), row groups are
// reduced through shared memory.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace la2 {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

constexpr int kDecThreads = 256;

// Shared memory: q and k of the sequence (d floats each) and one partial sum
// of 4 floats per thread.
inline size_t decode_smem_bytes(int d) {
    return sizeof(float) * (2 * static_cast<size_t>(d) + 4 * kDecThreads);
}

template <typename Tin, bool kVec>
__global__ void __launch_bounds__(kDecThreads)
la2_decode_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                  const float* __restrict__ decay, float* __restrict__ state,
                  float* __restrict__ out, int H, int d, int e)
{
    extern __shared__ float dsm[];
    float* qs = dsm;
    float* ks = dsm + d;
    float* part = dsm + 2 * d;  // [kDecThreads][4]
    const int n = blockIdx.x, tid = threadIdx.x;
    const float lam = decay[n % H];
    for (int i = tid; i < d; i += kDecThreads) {
        qs[i] = to_f32(q[static_cast<size_t>(n) * d + i]);
        ks[i] = to_f32(k[static_cast<size_t>(n) * d + i]);
    }
    __syncthreads();
    float* S = state + static_cast<size_t>(n) * d * e;
    const Tin* vn = v + static_cast<size_t>(n) * e;
    float* on = out + static_cast<size_t>(n) * e;
    constexpr int W = kVec ? 4 : 1;           // columns per thread
    const int ec = e / W;                     // column units
    for (int j0 = 0; j0 < ec; j0 += kDecThreads) {
        const int cu = min(ec - j0, kDecThreads);  // column units in this pass
        const int rgn = kDecThreads / cu;          // row groups
        const int ju = tid % cu, rg = tid / cu;
        const int col = (j0 + ju) * W;
        float acc[W], vv[W];
#pragma unroll
        for (int w = 0; w < W; ++w) {
            acc[w] = 0.f;
            vv[w] = to_f32(vn[col + w]);
        }
        // rows rg, rg + rgn, ...: kRows of them loaded before any is stored,
        // so that the loads of one thread are in flight together
        auto update_row = [&](int i, float (&sv)[W]) {
            const float ki = ks[i], qi = qs[i];
#pragma unroll
            for (int w = 0; w < W; ++w) {
                sv[w] = fmaf(lam, sv[w], ki * vv[w]);
                acc[w] = fmaf(sv[w], qi, acc[w]);
            }
        };
        auto load_row = [&](int i, float (&sv)[W]) {
            const float* row = S + static_cast<size_t>(i) * e + col;
            if constexpr (kVec) {
                const float4 s4 = *reinterpret_cast<const float4*>(row);
                sv[0] = s4.x; sv[1] = s4.y; sv[2] = s4.z; sv[3] = s4.w;
            } else {
                sv[0] = row[0];
            }
        };
        auto store_row = [&](int i, const float (&sv)[W]) {
            float* row = S + static_cast<size_t>(i) * e + col;
            if constexpr (kVec) *reinterpret_cast<float4*>(row) = make_float4(sv[0], sv[1], sv[2], sv[3]);
            else row[0] = sv[0];
        };
        if (rg < rgn) {
            constexpr int kRows = 4;
            int i = rg;
            for (; i + (kRows - 1) * rgn < d; i += kRows * rgn) {
                float sv[kRows][W];
#pragma unroll
                for (int b = 0; b < kRows; ++b) load_row(i + b * rgn, sv[b]);
#pragma unroll
                for (int b = 0; b < kRows; ++b) {
                    update_row(i + b * rgn, sv[b]);
                    store_row(i + b * rgn, sv[b]);
                }
            }
            for (; i < d; i += rgn) {
                float sv[W];
                load_row(i, sv);
                update_row(i, sv);
                store_row(i, sv);
            }
        }
#pragma unroll
        for (int w = 0; w < W; ++w) part[4 * tid + w] = acc[w];
        __syncthreads();
        if (tid < cu) {
#pragma unroll
            for (int w = 0; w < W; ++w) {
                float s = 0.f;
                for (int g = 0; g < rgn; ++g) s += part[4 * (g * cu + tid) + w];
                on[(j0 + tid) * W + w] = s;
            }
        }
        __syncthreads();
    }
}

}  // namespace la2
