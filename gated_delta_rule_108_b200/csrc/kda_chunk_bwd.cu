// kda_chunk_bwd.cu -- chunkwise KDA backward on CUDA cores in fp32 (sm_100a).
//
// The chunkwise form is the training mode of news.bugfactory.tech/news/3610
// (KDA paragraph); this file differentiates it.  The forward chunk algebra
// (unrolling the update equation of the daiw.net page, section "KDA 的更新式",
// over a chunk of L <= 64 tokens; g_r = sum_{i<=r} log_alpha_i per channel):
//
//   Kl = k e^{g-g_m}  Kr = k e^{g_m-g}  Ql = q e^{g-g_m}     (split at the middle token)
//   M = Kl Kr^T,  A = diag(beta) M (strictly lower),  P = Ql Kr^T (lower incl. diagonal)
//   T = (I + A)^{-1},  K~ = k e^{g},  Q~ = q e^{g},  K^ = k e^{g_{L-1}-g},  gamma = e^{g_{L-1}}
//   W = T diag(beta) K~,  U0 = T diag(beta) V
//   U = U0 - W S,  O = c (Q~ S + P U),  S' = Diag(gamma) S + K^^T U       (c = dk^{-1/2})
//
// Reverse, with D = c dO and dS' the cotangent of the state leaving the chunk:
//
//   across chunks (serial, reversed; KB3):
//     dU = P^T D + K^ dS'               dS = Diag(gamma) dS' + Q~^T D - W^T dU
//   within a chunk (all chunks in parallel; KB4):
//     dQ~ = D S^T   dK^ = U dS'^T   dW = -dU S^T   dP = D U^T (lower)   dgamma = rowsum(dS' * S)
//     Z = T^T dU  -> dv = beta Z,  dbeta += <Z, v>
//     Y = T^T dW  -> dK~ = beta Y, dbeta += <Y, K~>
//     dT = (dW K~^T + dU V^T) diag(beta);   dA = -T^T dT T^T (strictly lower)
//     dbeta += rowsum(dA * M);  dM = diag(beta) dA
//     dKl = dM Kr,  dQl = dP Kr,  dKr = dM^T Kl + dP^T Ql
//     dk = dKl e^{g-g_m} + dKr e^{g_m-g} + dK~ e^{g} + dK^ e^{g_{L-1}-g}
//     dq = dQl e^{g-g_m} + dQ~ e^{g}
//     dg = k (dKl e^{g-g_m} - dKr e^{g_m-g} + dK~ e^{g} - dK^ e^{g_{L-1}-g}) + q (dQl e^{g-g_m} + dQ~ e^{g})
//     dg_{L-1} += sum_r dK^_r K^_r + dgamma gamma;   dlog_alpha_s = sum_{r>=s} dg_r
//
// (The split point g_m cancels in M and P, so it carries no gradient.)  Chunks
// whose decay is too strong for the split factors use the exact pairwise form
// e^{g_r - g_i} <= 1 instead, as the forward does.
//
// The forward quantities come from the forward kernels run again with two
// extra outputs: T from K1 and the state entering every chunk from K2.
//
// These two kernels are the whole backward for fp32 inputs.  For bf16 inputs
// the tensor-core kernels (kda_chunk_tc.cu) compute the same quantities, and
// KB4 here reads their products and takes only the chunks that the forward
// kernel flagged as too strongly decayed for the split factors.
#include "kda_common.cuh"
#include "kda_launch.h"
#include "ptx.cuh"

namespace kda {
namespace {

constexpr float kMaxSplitExponent = 60.f;   // same split guard as the forward

template <int DK, int DV>
using Rec = F32Rec<DK, DV>;

// ------------------------------------------------------------------ KB3 ----
constexpr int kSlice = 64;   // value columns per CTA
constexpr int kInterThreads = 256;

// Shared memory of KB3.  The record tiles are unpadded copies of the record
// rows (every access below is a broadcast or along consecutive columns).
template <typename T, int DK>
struct BwdInterSmem {
    float dS[DK][kSlice + 1];
    float W[kChunk][DK];
    float Qt[kChunk][DK];
    float Kh[kChunk][DK];
    float P[kChunk][kChunk];
    float dU[kChunk][kSlice + 4];
    float gC[DK];
    T D[2][kChunk][kSlice];   // raw cotangent slice of o, double-buffered
};

template <typename T>
__device__ __forceinline__ float4 load4f(const T* p);
template <>
__device__ __forceinline__ float4 load4f<float>(const float* p) { return *reinterpret_cast<const float4*>(p); }
template <>
__device__ __forceinline__ float4 load4f<__nv_bfloat16>(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
}

// One CTA (8 warps) per (sequence, head, 64-wide value slice), serial over the
// chunks in reverse.  The loads of chunk n-1 are software-pipelined with the
// work of chunk n: K^, P and the cotangent slice are fetched (cp.async) as soon
// as step 1 of chunk n is done with them, Q~, W and gamma as soon as step 2 is.
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kInterThreads, 1)
bwd_inter_kernel(const T* __restrict__ d_o, const float* __restrict__ d_final_state,
                 float* __restrict__ d_initial_state, float* __restrict__ dS_end, float* __restrict__ dU_all,
                 ChunkMap map, const WsHeader* __restrict__ hdr, const float* __restrict__ records,
                 int H, size_t max_chunks, float scale)
{
    using R = Rec<DK, DV>;
    using Sm = BwdInterSmem<T, DK>;
    constexpr int NT = kInterThreads;
    constexpr int CPT = kSlice * DK / NT;   // step-2 columns per thread
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Sm& sm = *reinterpret_cast<Sm*>(smem_raw);

    if (hdr->status != kStatusOk) return;
    const int s = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * kSlice;
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    const size_t state_off = ((size_t)s * H + h) * DK * DV;

    for (int idx = tid; idx < DK * kSlice; idx += NT) {
        const int r = idx / kSlice, j = idx - r * kSlice;
        sm.dS[r][j] = d_final_state ? d_final_state[state_off + (size_t)r * DV + j0 + j] : 0.f;
    }
    const int first = map.seq_first_chunk(s);
    const int nch = map.seq_num_chunks(s);
    const int tok_begin = map.seq_token_begin(s), tok_end = map.seq_token_end(s);

    auto issue_a = [&](int n) {   // K^, P, cotangent slice of chunk n
        const float* rec = records + ((size_t)h * max_chunks + first + n) * R::FLOATS;
        for (int e = tid; e < kChunk * DK / 4; e += NT) ptx::cp_async16(&sm.Kh[0][0] + 4 * e, rec + R::KH + 4 * e);
        for (int e = tid; e < kChunk * kChunk / 4; e += NT) ptx::cp_async16(&sm.P[0][0] + 4 * e, rec + R::P + 4 * e);
        constexpr int EPP = 16 / (int)sizeof(T);   // elements per 16-byte piece
        constexpr int PPR = kSlice / EPP;          // pieces per row
        const int tok0 = tok_begin + n * kChunk;
        for (int e = tid; e < kChunk * PPR; e += NT) {
            const int r = e / PPR, pc = e - r * PPR;
            const bool live = tok0 + r < tok_end;   // rows past the sequence are zero-filled
            const T* src = d_o + ((size_t)(live ? tok0 + r : tok0) * H + h) * DV + j0 + pc * EPP;
            ptx::cp_async16(&sm.D[n & 1][r][pc * EPP], src, live ? 16u : 0u);
        }
    };
    auto issue_b = [&](int n) {   // Q~, W, gamma of chunk n
        const float* rec = records + ((size_t)h * max_chunks + first + n) * R::FLOATS;
        for (int e = tid; e < kChunk * DK / 4; e += NT) {
            ptx::cp_async16(&sm.Qt[0][0] + 4 * e, rec + R::QT + 4 * e);
            ptx::cp_async16(&sm.W[0][0] + 4 * e, rec + R::W + 4 * e);
        }
        for (int e = tid; e < DK / 4; e += NT) ptx::cp_async16(&sm.gC[0] + 4 * e, rec + R::GC + 4 * e);
    };

    if (nch > 0) {
        issue_a(nch - 1);
        ptx::cp_async_commit();
        issue_b(nch - 1);
        ptx::cp_async_commit();
    }
    for (int n = nch - 1; n >= 0; --n) {
        const size_t item = (size_t)h * max_chunks + first + n;
        const int buf = n & 1;
        ptx::cp_async_wait<1>();   // this thread's part of K^, P, D of chunk n has landed
        __syncthreads();           // everyone's; dS of the chunk after this one is complete
        {
            float* out = dS_end + item * DK * DV;
            for (int idx = tid; idx < DK * kSlice; idx += NT) {
                const int r = idx / kSlice, j = idx - r * kSlice;
                out[(size_t)r * DV + j0 + j] = sm.dS[r][j];
            }
        }

        // 1. dU = P^T D + K^ dS' for rows r = wp + 8a, columns lane and lane + 32
        float acc[8][2];
#pragma unroll
        for (int a = 0; a < 8; ++a) { acc[a][0] = 0.f; acc[a][1] = 0.f; }
        for (int c = 0; c < DK; c += 4) {
            float s0[4], s1[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) { s0[t] = sm.dS[c + t][lane]; s1[t] = sm.dS[c + t][lane + 32]; }
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const float4 kh = *reinterpret_cast<const float4*>(&sm.Kh[wp + 8 * a][c]);
                acc[a][0] += kh.x * s0[0] + kh.y * s0[1] + kh.z * s0[2] + kh.w * s0[3];
                acc[a][1] += kh.x * s1[0] + kh.y * s1[1] + kh.z * s1[2] + kh.w * s1[3];
            }
        }
        for (int i = 0; i < kChunk; ++i) {
            const float d0 = scale * to_f32(sm.D[buf][i][lane]);
            const float d1 = scale * to_f32(sm.D[buf][i][lane + 32]);
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const float p = sm.P[i][wp + 8 * a];
                acc[a][0] = fmaf(p, d0, acc[a][0]);
                acc[a][1] = fmaf(p, d1, acc[a][1]);
            }
        }
        {
            float* out = dU_all + item * kChunk * DV;
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const int r = wp + 8 * a;
                sm.dU[r][lane] = acc[a][0];
                sm.dU[r][lane + 32] = acc[a][1];
                out[(size_t)r * DV + j0 + lane] = acc[a][0];
                out[(size_t)r * DV + j0 + lane + 32] = acc[a][1];
            }
        }
        __syncthreads();   // K^ and P are free, dU is complete
        if (n > 0) {
            issue_a(n - 1);
            ptx::cp_async_commit();
            ptx::cp_async_wait<1>();   // Q~, W, gamma of chunk n have landed
        } else {
            ptx::cp_async_wait<0>();
        }
        __syncthreads();

        // 2. dS = Diag(gamma) dS' + Q~^T D - W^T dU: key row c, CPT columns from jb
        {
            const int c = tid % DK, jb = (tid / DK) * CPT;
            float x[CPT];
            const float gc = sm.gC[c];
#pragma unroll
            for (int j = 0; j < CPT; ++j) x[j] = gc * sm.dS[c][jb + j];
            for (int r = 0; r < kChunk; ++r) {
                const float qt = scale * sm.Qt[r][c], w = sm.W[r][c];
#pragma unroll
                for (int j = 0; j < CPT; j += 4) {
                    const float4 d = load4f<T>(&sm.D[buf][r][jb + j]);
                    const float4 u = *reinterpret_cast<const float4*>(&sm.dU[r][jb + j]);
                    x[j] += qt * d.x - w * u.x;
                    x[j + 1] += qt * d.y - w * u.y;
                    x[j + 2] += qt * d.z - w * u.z;
                    x[j + 3] += qt * d.w - w * u.w;
                }
            }
#pragma unroll
            for (int j = 0; j < CPT; ++j) sm.dS[c][jb + j] = x[j];   // this thread's own segment
        }
        __syncthreads();   // Q~, W and this chunk's D are free
        if (n > 0) {
            issue_b(n - 1);
            ptx::cp_async_commit();
        }
    }
    __syncthreads();
    if (d_initial_state) {
        for (int idx = tid; idx < DK * kSlice; idx += NT) {
            const int r = idx / kSlice, j = idx - r * kSlice;
            d_initial_state[state_off + (size_t)r * DV + j0 + j] = sm.dS[r][j];
        }
    }
}

// ------------------------------------------------------------------ KB4 ----
// A 64 x N product for the whole CTA (256 threads): thread (ty, tx) = (tid/16,
// tid%16) owns rows 4 ty .. 4 ty + 3 and columns 64 h + 4 tx .. + 3 (h < N/64).
// Operands are fp32 matrices in global memory (L2-resident scratch or inputs),
// read in K-slabs of 32 through shared memory.  Element (r, c) of a Mat is
// p[r * ld + c], or p[c * ld + r] when t is set (the stored matrix transposed).
struct Mat {
    const float* p;
    int ld;
    bool t;
    __device__ __forceinline__ float at(int r, int c) const {
        return t ? p[(size_t)c * ld + r] : p[(size_t)r * ld + c];
    }
};

constexpr int kSlab = 32;
constexpr int kMaxN = 128;

struct GemmStage {
    float a[kSlab][64 + 4];
    float b[kSlab][kMaxN + 4];
};

template <int N>
__device__ __forceinline__ void zero_acc(float (&acc)[4][N / 16]) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < N / 16; ++j) acc[i][j] = 0.f;
}

// acc += A(64 x K) B(K x N).  Each K-slab is read with 16-byte loads along the
// stored matrix's contiguous dimension into registers one slab ahead, so the
// L2 latency of slab s+1 overlaps the products of slab s; the stage holds the
// slab as a[k][m] and b[k][n] whatever the stored orientation.
template <int N>
__device__ void gemm64(float (&acc)[4][N / 16], Mat A, Mat B, int K, GemmStage& st) {
    constexpr int A4 = 64 * kSlab / 4 / 256;   // float4s of the A slab per thread
    constexpr int B4 = N * kSlab / 4 / 256;
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    float4 ra[A4], rb[B4];
    auto load = [&](int k0) {
#pragma unroll
        for (int i = 0; i < A4; ++i) {
            const int e = tid + 256 * i;
            ra[i] = A.t ? *reinterpret_cast<const float4*>(A.p + (size_t)(k0 + (e >> 4)) * A.ld + (e & 15) * 4)
                        : *reinterpret_cast<const float4*>(A.p + (size_t)(e >> 3) * A.ld + k0 + (e & 7) * 4);
        }
#pragma unroll
        for (int i = 0; i < B4; ++i) {
            const int e = tid + 256 * i;
            rb[i] = B.t ? *reinterpret_cast<const float4*>(B.p + (size_t)(e >> 3) * B.ld + k0 + (e & 7) * 4)
                        : *reinterpret_cast<const float4*>(B.p + (size_t)(k0 + e / (N / 4)) * B.ld + (e % (N / 4)) * 4);
        }
    };
    auto store = [&]() {
#pragma unroll
        for (int i = 0; i < A4; ++i) {
            const int e = tid + 256 * i;
            if (A.t) {
                *reinterpret_cast<float4*>(&st.a[e >> 4][(e & 15) * 4]) = ra[i];
            } else {
                const int m = e >> 3, k4 = (e & 7) * 4;
                st.a[k4][m] = ra[i].x; st.a[k4 + 1][m] = ra[i].y;
                st.a[k4 + 2][m] = ra[i].z; st.a[k4 + 3][m] = ra[i].w;
            }
        }
#pragma unroll
        for (int i = 0; i < B4; ++i) {
            const int e = tid + 256 * i;
            if (B.t) {
                const int n = e >> 3, k4 = (e & 7) * 4;
                st.b[k4][n] = rb[i].x; st.b[k4 + 1][n] = rb[i].y;
                st.b[k4 + 2][n] = rb[i].z; st.b[k4 + 3][n] = rb[i].w;
            } else {
                *reinterpret_cast<float4*>(&st.b[e / (N / 4)][(e % (N / 4)) * 4]) = rb[i];
            }
        }
    };
    __syncthreads();   // operands written by earlier epilogues are complete
    load(0);
    for (int k0 = 0; k0 < K; k0 += kSlab) {
        __syncthreads();   // earlier readers of the stage are done
        store();
        __syncthreads();
        if (k0 + kSlab < K) load(k0 + kSlab);
#pragma unroll 4
        for (int kk = 0; kk < kSlab; ++kk) {
            const float4 av = *reinterpret_cast<const float4*>(&st.a[kk][ty * 4]);
            const float ar[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
            for (int hh = 0; hh < N / 64; ++hh) {
                const float4 bv = *reinterpret_cast<const float4*>(&st.b[kk][hh * 64 + tx * 4]);
                const float br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][hh * 4 + j] = fmaf(ar[i], br[j], acc[i][hh * 4 + j]);
            }
        }
    }
}

// f(row, col, value) over the thread's accumulators
template <int N, typename F>
__device__ __forceinline__ void for_acc(float (&acc)[4][N / 16], F f) {
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int hh = 0; hh < N / 64; ++hh)
#pragma unroll
            for (int j = 0; j < 4; ++j) f(ty * 4 + i, hh * 64 + tx * 4 + j, acc[i][hh * 4 + j]);
}

// Sum over the 16 threads that share a row (one half-warp).
__device__ __forceinline__ float row_sum16(float x) {
#pragma unroll
    for (int off = 8; off; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// Per-CTA fp32 scratch (global memory), offsets in floats.
template <int DK, int DV>
struct Scr {
    static constexpr size_t KL = 0;                     // k e^{g-g_m} (strong chunk: raw k)
    static constexpr size_t KR = KL + kChunk * DK;      // k e^{g_m-g}
    static constexpr size_t QL = KR + kChunk * DK;      // q e^{g-g_m} (strong chunk: raw q)
    static constexpr size_t KT = QL + kChunk * DK;      // K~ = k e^{g}
    static constexpr int DX = DK > DV ? DK : DV;       // value-side buffers are reused for 64 x DK
    static constexpr size_t VV = KT + kChunk * DK;      // v
    static constexpr size_t DO = VV + kChunk * DX;      // c dO
    static constexpr size_t U = DO + kChunk * DX;
    static constexpr size_t DQT = U + kChunk * DX;
    static constexpr size_t DKH = DQT + kChunk * DK;
    static constexpr size_t DW = DKH + kChunk * DK;
    static constexpr size_t DKT = DW + kChunk * DK;
    static constexpr size_t DP = DKT + kChunk * DK;
    static constexpr size_t DT = DP + kChunk * kChunk;
    static constexpr size_t X1 = DT;                    // dT T^T overwrites dT (read in full first)
    static constexpr size_t DM = DT + kChunk * kChunk;
    static constexpr size_t M = DM + kChunk * kChunk;
    static constexpr size_t FLOATS = M + kChunk * kChunk;
    // the last products reuse buffers that are dead by then (v, D and U are
    // last read by the dT and dP products)
    static constexpr size_t DKL = VV;                   // dKl e^{g-g_m}
    static constexpr size_t DQL = DO;                   // dQl e^{g-g_m}
    static constexpr size_t DKR = U;                    // dKr e^{g_m-g}
};

template <int DK>
struct BwdIntraSmem {
    GemmStage st;
    float g[kChunk][DK];   // cumulative log-decay, later dg
    float gm[DK], gl[DK], dgam[DK], dgl[DK];
    float beta[kChunk], dbeta[kChunk];
};

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(256, 2)
bwd_intra_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                 const float* __restrict__ log_alpha, const float* __restrict__ beta, const T* __restrict__ d_o,
                 ChunkMap map, const WsHeader* __restrict__ hdr, const float* __restrict__ records,
                 const float* __restrict__ tmat, const float* __restrict__ states,
                 const float* __restrict__ dS_end, const float* __restrict__ dU_all, float* scratch,
                 T* __restrict__ dq, T* __restrict__ dk, T* __restrict__ dv, float* __restrict__ dla,
                 float* __restrict__ dbeta, int H, size_t max_chunks, float scale, int gate,
                 const float* __restrict__ vside, const int* __restrict__ only_flagged)
{
    using R = Rec<DK, DV>;
    using C = Scr<DK, DV>;
    using Sm = BwdIntraSmem<DK>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Sm& sm = *reinterpret_cast<Sm*>(smem_raw);

    if (hdr->status != kStatusOk) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t rowk = (size_t)H * DK, rowv = (size_t)H * DV;
    const long total = (long)hdr->num_chunks * H;
    float* scr = scratch + (size_t)blockIdx.x * C::FLOATS;

    for (long item = blockIdx.x; item < total; item += gridDim.x) {
        const int c = (int)(item / H), h = (int)(item % H);
        // with the split-factor products on the tensor cores, only the chunks that
        // took the strong-decay (exact) path are left to this kernel
        if (only_flagged && !only_flagged[(size_t)h * max_chunks + c]) continue;
        int s, tok0, L;
        map.locate(c, s, tok0, L);
        const size_t it = (size_t)h * max_chunks + c;
        const float* rec = records + it * R::FLOATS;
        const float* Tm = tmat + it * kChunk * kChunk;
        const float* Sn = states + it * DK * DV;
        const float* dSe = dS_end + it * DK * DV;
        const float* dUc = dU_all + it * kChunk * DV;
        // the products over the value dimension: precomputed (bf16 inputs) or formed here
        const float* vs = vside ? vside + it * VSide<DK>::FLOATS : nullptr;
        const float* pDQT = vs ? vs + VSide<DK>::DQT : scr + C::DQT;
        const float* pDW = vs ? vs + VSide<DK>::DW : scr + C::DW;
        const float* pDKH = vs ? vs + VSide<DK>::DKH : scr + C::DKH;
        const float* pDP = vs ? vs + VSide<DK>::DP : scr + C::DP;

        __syncthreads();   // the previous item is done with shared memory and scratch
        // ---- cumulative log-decay, beta --------------------------------------
        if (tid < DK) {
            // per-channel gate [.., H, DK]; per-head gate [.., H] (the same value
            // for every channel); no gate: log-decay 0
            float acc = 0.f;
            if (gate == kGateNone) {
                for (int r = 0; r < kChunk; ++r) sm.g[r][tid] = 0.f;
            } else {
                const bool chan = gate == kGateChannel;
                const size_t rstride = chan ? rowk : (size_t)H;
                const float* la = chan ? log_alpha + (size_t)tok0 * rowk + (size_t)h * DK + tid
                                       : log_alpha + (size_t)tok0 * H + h;
#pragma unroll 16   // the loads are independent: keep 16 in flight
                for (int r = 0; r < kChunk; ++r) {
                    acc += (r < L) ? la[(size_t)r * rstride] : 0.f;
                    sm.g[r][tid] = acc;
                }
            }
            sm.dgl[tid] = 0.f;
        } else if (tid >= 128 && tid < 128 + kChunk) {
            const int r = tid - 128;
            sm.beta[r] = (r < L) ? beta[(size_t)(tok0 + r) * H + h] : 0.f;
            sm.dbeta[r] = vs ? vs[VSide<DK>::DBP + r] : 0.f;   // the parts through W, U0 when precomputed
        }
        __syncthreads();
        bool wide = false;
        if (tid < DK) {
            sm.gm[tid] = sm.g[(L - 1) >> 1][tid];
            sm.gl[tid] = sm.g[L - 1][tid];
            wide = fmaxf(sm.g[0][tid] - sm.gm[tid], sm.gm[tid] - sm.gl[tid]) > kMaxSplitExponent;
        }
        const bool strong = __syncthreads_or(wide);

        // ---- operands into scratch ------------------------------------------
#pragma unroll 4
        for (int idx = tid; idx < kChunk * DK; idx += 256) {
            const int r = idx / DK, ch = idx - r * DK;
            float kk = 0.f, qq = 0.f;
            if (r < L) {
                const size_t off = (size_t)(tok0 + r) * rowk + (size_t)h * DK + ch;
                kk = to_f32(k[off]);
                qq = to_f32(q[off]);
            }
            const float gg = sm.g[r][ch];
            if (!strong) {
                const float em = expf(gg - sm.gm[ch]);
                scr[C::KL + idx] = kk * em;
                scr[C::KR + idx] = kk * expf(sm.gm[ch] - gg);
                scr[C::QL + idx] = qq * em;
            } else {
                scr[C::KL + idx] = kk;
                scr[C::QL + idx] = qq;
            }
            if (!vs) scr[C::KT + idx] = kk * expf(gg);
        }
#pragma unroll 4
        for (int idx = tid; idx < kChunk * DV; idx += 256) {
            const int r = idx / DV, j = idx - r * DV;
            const size_t off = (size_t)(tok0 + r) * rowv + (size_t)h * DV + j;
            if (!vs) scr[C::VV + idx] = (r < L) ? to_f32(v[off]) : 0.f;
            if (!vs) scr[C::DO + idx] = (r < L) ? scale * to_f32(d_o[off]) : 0.f;
        }
        // dgamma_c = sum_j dS'_cj S_cj: one warp per key row
        if (vs) {
            if (tid < DK) sm.dgam[tid] = vs[VSide<DK>::DGAM + tid];
        } else
        for (int ch = warp; ch < DK; ch += 8) {
            float acc = 0.f;
            for (int j = lane; j < DV; j += 32) acc += dSe[(size_t)ch * DV + j] * Sn[(size_t)ch * DV + j];
#pragma unroll
            for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) sm.dgam[ch] = acc;
        }

        // ---- products over the value dimension ---------------------------------
        if (!vs) {
        {   // U = U0 - W S
            float acc[4][DV / 16];
            zero_acc<DV>(acc);
            gemm64<DV>(acc, Mat{rec + R::W, DK, false}, Mat{Sn, DV, false}, DK, sm.st);
            for_acc<DV>(acc, [&](int r, int n, float x) { scr[C::U + r * DV + n] = rec[R::U0 + r * DV + n] - x; });
        }
        {   // dQ~ = D S^T
            float acc[4][DK / 16];
            zero_acc<DK>(acc);
            gemm64<DK>(acc, Mat{scr + C::DO, DV, false}, Mat{Sn, DV, true}, DV, sm.st);
            for_acc<DK>(acc, [&](int r, int n, float x) { scr[C::DQT + r * DK + n] = x; });
        }
        {   // dW = -dU S^T
            float acc[4][DK / 16];
            zero_acc<DK>(acc);
            gemm64<DK>(acc, Mat{dUc, DV, false}, Mat{Sn, DV, true}, DV, sm.st);
            for_acc<DK>(acc, [&](int r, int n, float x) { scr[C::DW + r * DK + n] = -x; });
        }
        {   // dK^ = U dS'^T
            float acc[4][DK / 16];
            zero_acc<DK>(acc);
            gemm64<DK>(acc, Mat{scr + C::U, DV, false}, Mat{dSe, DV, true}, DV, sm.st);
            for_acc<DK>(acc, [&](int r, int n, float x) { scr[C::DKH + r * DK + n] = x; });
        }
        {   // dP = D U^T, lower triangle with the diagonal
            float acc[4][kChunk / 16];
            zero_acc<kChunk>(acc);
            gemm64<kChunk>(acc, Mat{scr + C::DO, DV, false}, Mat{scr + C::U, DV, true}, DV, sm.st);
            for_acc<kChunk>(acc, [&](int r, int i, float x) { scr[C::DP + r * kChunk + i] = (i <= r) ? x : 0.f; });
        }
        }   // !vs
        // ---- through W = T diag(beta) K~ and U0 = T diag(beta) V -------------
        // (precomputed on the tensor cores for bf16 inputs: dv, dK~, dA, dbeta parts)
        if (!vs) {
        {   // Z = T^T dU: dv = beta Z, dbeta += <Z, v>
            float acc[4][DV / 16];
            zero_acc<DV>(acc);
            gemm64<DV>(acc, Mat{Tm, kChunk, true}, Mat{dUc, DV, false}, kChunk, sm.st);
            float part[4] = {0.f, 0.f, 0.f, 0.f};
            for_acc<DV>(acc, [&](int r, int n, float x) {
                part[r & 3] += x * scr[C::VV + r * DV + n];
                if (r < L) dv[(size_t)(tok0 + r) * rowv + (size_t)h * DV + n] = from_f32<T>(sm.beta[r] * x);
            });
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float t = row_sum16(part[i]);
                if ((tid & 15) == 0) sm.dbeta[(tid >> 4) * 4 + i] += t;
            }
        }
        {   // Y = T^T dW: dK~ = beta Y, dbeta += <Y, K~>
            float acc[4][DK / 16];
            zero_acc<DK>(acc);
            gemm64<DK>(acc, Mat{Tm, kChunk, true}, Mat{pDW, DK, false}, kChunk, sm.st);
            float part[4] = {0.f, 0.f, 0.f, 0.f};
            for_acc<DK>(acc, [&](int r, int n, float x) {
                part[r & 3] += x * scr[C::KT + r * DK + n];
                scr[C::DKT + r * DK + n] = sm.beta[r] * x;
            });
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float t = row_sum16(part[i]);
                if ((tid & 15) == 0) sm.dbeta[(tid >> 4) * 4 + i] += t;
            }
        }
        {   // dT = (dW K~^T + dU V^T) diag(beta)
            float acc[4][kChunk / 16];
            zero_acc<kChunk>(acc);
            gemm64<kChunk>(acc, Mat{pDW, DK, false}, Mat{scr + C::KT, DK, true}, DK, sm.st);
            gemm64<kChunk>(acc, Mat{dUc, DV, false}, Mat{scr + C::VV, DV, true}, DV, sm.st);
            for_acc<kChunk>(acc, [&](int r, int i, float x) { scr[C::DT + r * kChunk + i] = x * sm.beta[i]; });
        }
        {   // X1 = dT T^T
            float acc[4][kChunk / 16];
            zero_acc<kChunk>(acc);
            gemm64<kChunk>(acc, Mat{scr + C::DT, kChunk, false}, Mat{Tm, kChunk, true}, kChunk, sm.st);
            for_acc<kChunk>(acc, [&](int r, int i, float x) { scr[C::X1 + r * kChunk + i] = x; });
        }
        }   // !vs
        // ---- M = Kl Kr^T (the unweighted A), strictly lower -------------------
        if (!strong) {
            float acc[4][kChunk / 16];
            zero_acc<kChunk>(acc);
            gemm64<kChunk>(acc, Mat{scr + C::KL, DK, false}, Mat{scr + C::KR, DK, true}, DK, sm.st);
            for_acc<kChunk>(acc, [&](int r, int i, float x) { scr[C::M + r * kChunk + i] = (i < r) ? x : 0.f; });
        } else {   // exact: one warp per (r, i), every exponent <= 0
            __syncthreads();
            for (int pr = warp; pr < kChunk * kChunk; pr += 8) {
                const int r = pr >> 6, i = pr & 63;
                float acc = 0.f;
                if (i < r)
                    for (int ch = lane; ch < DK; ch += 32)
                        acc += scr[C::KL + r * DK + ch] * scr[C::KL + i * DK + ch] * expf(sm.g[r][ch] - sm.g[i][ch]);
#pragma unroll
                for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                if (lane == 0) scr[C::M + pr] = acc;
            }
        }
        if (vs) {   // dA precomputed: dbeta += rowsum(dA M); dM = diag(beta) dA (one warp per row)
            __syncthreads();   // M complete
            for (int r = warp; r < kChunk; r += 8) {
                float part = 0.f;
#pragma unroll
                for (int i = lane; i < kChunk; i += 32) {
                    const float da = vs[VSide<DK>::DA + r * kChunk + i];
                    part += da * scr[C::M + r * kChunk + i];
                    scr[C::DM + r * kChunk + i] = sm.beta[r] * da;
                }
#pragma unroll
                for (int off = 16; off; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
                if (lane == 0) sm.dbeta[r] += part;
            }
        } else {   // dA = -T^T X1 (strictly lower); dbeta += rowsum(dA M); dM = diag(beta) dA
            float acc[4][kChunk / 16];
            zero_acc<kChunk>(acc);
            gemm64<kChunk>(acc, Mat{Tm, kChunk, true}, Mat{scr + C::X1, kChunk, false}, kChunk, sm.st);
            float part[4] = {0.f, 0.f, 0.f, 0.f};
            for_acc<kChunk>(acc, [&](int r, int i, float x) {
                const float da = (i < r) ? -x : 0.f;
                part[r & 3] += da * scr[C::M + r * kChunk + i];
                scr[C::DM + r * kChunk + i] = sm.beta[r] * da;
            });
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float t = row_sum16(part[i]);
                if ((tid & 15) == 0) sm.dbeta[(tid >> 4) * 4 + i] += t;
            }
        }
        // ---- through M and P to the (decayed) keys and queries ---------------
        if (!strong) {
            {   // dKl = dM Kr, dQl = dP Kr (times e^{g-g_m})
                float acc[4][DK / 16];
                zero_acc<DK>(acc);
                gemm64<DK>(acc, Mat{scr + C::DM, kChunk, false}, Mat{scr + C::KR, DK, false}, kChunk, sm.st);
                for_acc<DK>(acc, [&](int r, int n, float x) {
                    scr[C::DKL + r * DK + n] = x * expf(sm.g[r][n] - sm.gm[n]);
                });
                zero_acc<DK>(acc);
                gemm64<DK>(acc, Mat{pDP, kChunk, false}, Mat{scr + C::KR, DK, false}, kChunk, sm.st);
                for_acc<DK>(acc, [&](int r, int n, float x) {
                    scr[C::DQL + r * DK + n] = x * expf(sm.g[r][n] - sm.gm[n]);
                });
            }
            {   // dKr = dM^T Kl + dP^T Ql (times e^{g_m-g})
                float acc[4][DK / 16];
                zero_acc<DK>(acc);
                gemm64<DK>(acc, Mat{scr + C::DM, kChunk, true}, Mat{scr + C::KL, DK, false}, kChunk, sm.st);
                gemm64<DK>(acc, Mat{pDP, kChunk, true}, Mat{scr + C::QL, DK, false}, kChunk, sm.st);
                for_acc<DK>(acc, [&](int r, int n, float x) {
                    scr[C::DKR + r * DK + n] = x * expf(sm.gm[n] - sm.g[r][n]);
                });
            }
        } else {   // exact pairwise form; KL / QL hold the raw k / q
            __syncthreads();
            for (int idx = tid; idx < kChunk * DK; idx += 256) {
                const int r = idx / DK, ch = idx - r * DK;
                const float gr = sm.g[r][ch];
                const float kr = scr[C::KL + idx], qr = scr[C::QL + idx];
                float dkl = 0.f, dql = 0.f, dkr = 0.f;
                for (int i = 0; i <= r; ++i) {   // r is the later token
                    const float e = expf(gr - sm.g[i][ch]);
                    const float ki = scr[C::KL + i * DK + ch];
                    dql += pDP[r * kChunk + i] * ki * e;
                    if (i < r) dkl += scr[C::DM + r * kChunk + i] * ki * e;
                }
                for (int j = r; j < kChunk; ++j) {   // r is the earlier token
                    const float e = expf(sm.g[j][ch] - gr);
                    dkr += pDP[j * kChunk + r] * scr[C::QL + j * DK + ch] * e;
                    if (j > r) dkr += scr[C::DM + j * kChunk + r] * scr[C::KL + j * DK + ch] * e;
                }
                (void)kr; (void)qr;
                scr[C::DKL + idx] = dkl;
                scr[C::DQL + idx] = dql;
                scr[C::DKR + idx] = dkr;
            }
        }
        __syncthreads();

        // ---- dq, dk, dg -------------------------------------------------------
#pragma unroll 4
        for (int idx = tid; idx < kChunk * DK; idx += 256) {
            const int r = idx / DK, ch = idx - r * DK;
            float kk = 0.f, qq = 0.f;
            const size_t off = (size_t)(tok0 + r) * rowk + (size_t)h * DK + ch;
            if (r < L) {
                kk = to_f32(k[off]);
                qq = to_f32(q[off]);
            }
            const float gg = sm.g[r][ch];
            const float eg = expf(gg), eh = expf(sm.gl[ch] - gg);
            const float dkl = scr[C::DKL + idx], dkr = scr[C::DKR + idx], dql = scr[C::DQL + idx];
            const float dkt = vs ? vs[VSide<DK>::DKT + idx] : scr[C::DKT + idx], dkh = pDKH[idx], dqt = pDQT[idx];
            if (r < L) {
                dk[off] = from_f32<T>(dkl + dkr + dkt * eg + dkh * eh);
                dq[off] = from_f32<T>(dql + dqt * eg);
            }
            const float kh = kk * eh;
            atomicAdd(&sm.dgl[ch], dkh * kh);
            sm.g[r][ch] = kk * (dkl - dkr + dkt * eg) - dkh * kh + qq * (dql + dqt * eg);   // dg
        }
        __syncthreads();
        // dlog_alpha_s = sum_{r >= s} dg_r, with g_{L-1}'s own cotangent added at
        // L-1; a per-head gate is shared by all channels, so its cotangent is
        // the sum over channels
        if (gate != kGateNone && tid < DK) {
            float run = sm.dgl[tid] + sm.dgam[tid] * expf(sm.gl[tid]);
            for (int r = L - 1; r >= 0; --r) {
                run += sm.g[r][tid];
                if (gate == kGateChannel) dla[(size_t)(tok0 + r) * rowk + (size_t)h * DK + tid] = run;
                else sm.g[r][tid] = run;
            }
        }
        if (tid >= 128 && tid < 128 + kChunk) {
            const int r = tid - 128;
            if (r < L) dbeta[(size_t)(tok0 + r) * H + h] = sm.dbeta[r];
        }
        if (gate == kGateHead) {
            __syncthreads();
            if (tid < L) {
                float acc = 0.f;
                for (int c = 0; c < DK; ++c) acc += sm.g[tid][(c + tid) % DK];   // rotated: no bank conflicts
                dla[(size_t)(tok0 + tid) * H + h] = acc;
            }
        }
    }
}

template <typename T, int DK, int DV>
cudaError_t launch_bwd_inter_t(const ChunkArgs& a) {
    ChunkMap map{a.cu_seqlens, a.chunk_offsets, a.num_seqs, a.T, a.fixed_chunks_per_seq};
    auto kern = bwd_inter_kernel<T, DK, DV>;
    const int smem = (int)sizeof(BwdInterSmem<T, DK>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)a.num_seqs, (unsigned)a.H, (unsigned)(DV / kSlice));
    kern<<<grid, kInterThreads, smem, a.stream>>>(static_cast<const T*>(a.d_o), a.d_final_state, a.d_initial_state,
                                         a.dS_end, a.dU, map, static_cast<const WsHeader*>(a.ws_header),
                                         static_cast<const float*>(a.records), a.H, a.max_chunks, a.scale);
    return cudaGetLastError();
}

template <typename T, int DK, int DV>
cudaError_t launch_bwd_intra_t(const ChunkArgs& a) {
    if (a.max_chunks == 0 || a.bwd_ctas <= 0) return cudaSuccess;
    ChunkMap map{a.cu_seqlens, a.chunk_offsets, a.num_seqs, a.T, a.fixed_chunks_per_seq};
    auto kern = bwd_intra_kernel<T, DK, DV>;
    const int smem = (int)sizeof(BwdIntraSmem<DK>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<a.bwd_ctas, 256, smem, a.stream>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v), a.log_alpha, a.beta,
        static_cast<const T*>(a.d_o), map, static_cast<const WsHeader*>(a.ws_header),
        static_cast<const float*>(a.records), a.tmat, a.states, a.dS_end, a.dU, a.scratch,
        static_cast<T*>(a.dq), static_cast<T*>(a.dk_out), static_cast<T*>(a.dv_out), a.dlog_alpha, a.dbeta,
        a.H, a.max_chunks, a.scale, a.gate, a.vside, a.bwd_flags);
    return cudaGetLastError();
}

#define KDA_BWD_DISPATCH(FN, a)                                                     \
    do {                                                                            \
        if ((a).bf16) {                                                             \
            if ((a).dk == 128 && (a).dv == 128) return FN<__nv_bfloat16, 128, 128>(a); \
            if ((a).dk == 128 && (a).dv == 64) return FN<__nv_bfloat16, 128, 64>(a);   \
            if ((a).dk == 64 && (a).dv == 128) return FN<__nv_bfloat16, 64, 128>(a);   \
            if ((a).dk == 64 && (a).dv == 64) return FN<__nv_bfloat16, 64, 64>(a);     \
        } else {                                                                    \
            if ((a).dk == 128 && (a).dv == 128) return FN<float, 128, 128>(a);         \
            if ((a).dk == 128 && (a).dv == 64) return FN<float, 128, 64>(a);           \
            if ((a).dk == 64 && (a).dv == 128) return FN<float, 64, 128>(a);           \
            if ((a).dk == 64 && (a).dv == 64) return FN<float, 64, 64>(a);             \
        }                                                                           \
        return cudaErrorInvalidValue;                                               \
    } while (0)

}  // namespace

size_t bwd_scratch_bytes_per_cta(int dk, int dv) {
    if (dk == 128 && dv == 128) return Scr<128, 128>::FLOATS * sizeof(float);
    if (dk == 128 && dv == 64) return Scr<128, 64>::FLOATS * sizeof(float);
    if (dk == 64 && dv == 128) return Scr<64, 128>::FLOATS * sizeof(float);
    if (dk == 64 && dv == 64) return Scr<64, 64>::FLOATS * sizeof(float);
    return 0;
}

cudaError_t launch_chunk_bwd_inter(const ChunkArgs& a) {
    if (a.num_seqs == 0) return cudaSuccess;
    KDA_BWD_DISPATCH(launch_bwd_inter_t, a);
}

cudaError_t launch_chunk_bwd_intra(const ChunkArgs& a) { KDA_BWD_DISPATCH(launch_bwd_intra_t, a); }

}  // namespace kda
