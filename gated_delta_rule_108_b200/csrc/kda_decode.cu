// kda_decode.cu -- one-token KDA step for B x H independent states (sm_100a).
//
// "Fused recurrent" mode of news.bugfactory.tech/news/3610 (KDA paragraph):
// every (sequence, head) state tile is read once from HBM, updated by one
// token and written back once.  Per head, with S in R^{dk x dv} (rows = key
// channels), the daiw.net update equation (section "KDA 的更新式") is applied
// in the forget -> predict -> correct -> write -> read order:
//
//   S~ = Diag(alpha) S          p = S~^T k          u = beta (v - p)
//   S' = S~ + k u^T             o = dk^{-1/2} S'^T q = dk^{-1/2} (S~^T q + u <k, q>)
//
// The last identity lets the read share the pass over S~ with the predict, so
// S is touched by exactly one load and one store per element.  With a per-head
// gate (Gated DeltaNet) every channel decays by the same alpha; without a gate
// (DeltaNet) alpha = 1.
//
// Layout: one CTA per (b, h); warp w owns key rows [w*DK/NW, (w+1)*DK/NW), lane
// l owns value columns [l*DV/32, (l+1)*DV/32) -- a warp reads one 512-byte row
// per 128-bit load instruction at dv = 128.  Column sums over rows (p and
// S~^T q) are combined across warps through shared memory; <k, q> is a warp
// shuffle reduction.  The state is bandwidth-bound traffic with no reuse, so
// it is loaded/stored with the streaming cache hint.
#include "kda_common.cuh"
#include "kda_launch.h"

namespace kda {
namespace {

template <int VEC> struct VecT;
template <> struct VecT<4> { using type = float4; };
template <> struct VecT<2> { using type = float2; };

template <int VEC>
__device__ __forceinline__ void load_vec(const float* p, float (&x)[VEC]) {
    if constexpr (VEC == 4) {
        const float4 t = __ldcs(reinterpret_cast<const float4*>(p));
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    } else {
        const float2 t = __ldcs(reinterpret_cast<const float2*>(p));
        x[0] = t.x; x[1] = t.y;
    }
}
template <int VEC>
__device__ __forceinline__ void store_vec(float* p, const float (&x)[VEC]) {
    if constexpr (VEC == 4) {
        __stcs(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
    } else {
        __stcs(reinterpret_cast<float2*>(p), make_float2(x[0], x[1]));
    }
}

template <typename T, int DK, int DV, int NW>
__global__ void __launch_bounds__(NW * 32)
decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   const float* __restrict__ log_alpha, const float* __restrict__ beta,
                   float* __restrict__ state, T* __restrict__ o, float scale, int gate)
{
    constexpr int NT = NW * 32;
    constexpr int ROWS = DK / NW;   // key rows per warp
    constexpr int VEC = DV / 32;    // value columns per lane
    static_assert(DK % NW == 0 && (VEC == 4 || VEC == 2), "tile shape");

    __shared__ float sk[DK], sq[DK], sa[DK], sv[DV], su[DV];
    __shared__ float red_p[NW][DV], red_q[NW][DV];
    __shared__ float s_kq;

    const int bh = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float* S = state + (size_t)bh * DK * DV;

    // The state tile is the only large read: issue all of it first.
    float s[ROWS][VEC];
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
        load_vec<VEC>(S + (size_t)(warp * ROWS + r) * DV + lane * VEC, s[r]);

    const float a_head = (gate == kGateHead) ? expf(log_alpha[bh]) : 1.f;
    for (int i = tid; i < DK; i += NT) {
        sk[i] = to_f32(k[(size_t)bh * DK + i]);
        sq[i] = to_f32(q[(size_t)bh * DK + i]);
        sa[i] = (gate == kGateChannel) ? expf(log_alpha[(size_t)bh * DK + i]) : a_head;
    }
    for (int j = tid; j < DV; j += NT) sv[j] = to_f32(v[(size_t)bh * DV + j]);
    __syncthreads();

    if (warp == 0) {
        float acc = 0.f;
        for (int i = lane; i < DK; i += 32) acc += sk[i] * sq[i];
#pragma unroll
        for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) s_kq = acc;
    }

    // forget, then partial column sums of S~^T k (predict) and S~^T q (read)
    float p[VEC], qs[VEC];
#pragma unroll
    for (int c = 0; c < VEC; ++c) { p[c] = 0.f; qs[c] = 0.f; }
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
        const int i = warp * ROWS + r;
        const float a = sa[i], ki = sk[i], qi = sq[i];
#pragma unroll
        for (int c = 0; c < VEC; ++c) {
            s[r][c] *= a;
            p[c] = fmaf(s[r][c], ki, p[c]);
            qs[c] = fmaf(s[r][c], qi, qs[c]);
        }
    }
#pragma unroll
    for (int c = 0; c < VEC; ++c) {
        red_p[warp][lane * VEC + c] = p[c];
        red_q[warp][lane * VEC + c] = qs[c];
    }
    __syncthreads();

    // correct (u = beta (v - p)) and read (o)
    const float b = beta[bh];
    for (int j = tid; j < DV; j += NT) {
        float pj = 0.f, qj = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) { pj += red_p[w][j]; qj += red_q[w][j]; }
        const float u = b * (sv[j] - pj);
        su[j] = u;
        o[(size_t)bh * DV + j] = from_f32<T>(scale * fmaf(u, s_kq, qj));
    }
    __syncthreads();

    // write: S' = S~ + k u^T
    float uu[VEC];
#pragma unroll
    for (int c = 0; c < VEC; ++c) uu[c] = su[lane * VEC + c];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
        const float ki = sk[warp * ROWS + r];
#pragma unroll
        for (int c = 0; c < VEC; ++c) s[r][c] = fmaf(ki, uu[c], s[r][c]);
        store_vec<VEC>(S + (size_t)(warp * ROWS + r) * DV + lane * VEC, s[r]);
    }
}

template <typename T, int DK, int DV>
cudaError_t launch_decode_t(const DecodeArgs& a) {
    constexpr int NW = 8;
    const int grid = a.B * a.H;
    decode_step_kernel<T, DK, DV, NW><<<grid, NW * 32, 0, a.stream>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v),
        a.log_alpha, a.beta, a.state, static_cast<T*>(a.o), a.scale, a.gate);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_decode_dt(const DecodeArgs& a) {
    if (a.dk == 128 && a.dv == 128) return launch_decode_t<T, 128, 128>(a);
    if (a.dk == 128 && a.dv == 64) return launch_decode_t<T, 128, 64>(a);
    if (a.dk == 64 && a.dv == 128) return launch_decode_t<T, 64, 128>(a);
    if (a.dk == 64 && a.dv == 64) return launch_decode_t<T, 64, 64>(a);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a) {
    if (a.B * a.H == 0) return cudaSuccess;
    return a.bf16 ? launch_decode_dt<__nv_bfloat16>(a) : launch_decode_dt<float>(a);
}

}  // namespace kda
