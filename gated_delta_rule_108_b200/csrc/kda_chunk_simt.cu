// kda_chunk_simt.cu -- chunkwise KDA forward on CUDA cores in fp32 (sm_100a).
//
// This is the fp32 path of kda_chunk_fwd: every product is an fp32 FMA, so it
// meets a 1e-4 relative error bound on fp32 inputs.  It implements the same
// chunk algebra as the tensor-core path, in three launches:
//
//   K0 chunk_prep   -- resets the workspace status; for packed sequences it
//                      checks cu_seqlens and builds the chunk table.
//   K1 intra_chunk  -- one CTA per (chunk, head), all chunks in parallel.
//   K2 inter_chunk  -- one CTA per (sequence, head, 64-wide value slice),
//                      serial over the sequence's chunks, state in shared memory.
//
// Chunk algebra (derived by unrolling the update equation of the daiw.net page,
// section "KDA 的更新式", over one chunk of L <= 64 tokens; S is the state
// entering the chunk, g_r = sum_{i<=r} log_alpha_i per key channel):
//
//   Q~_r = q_r e^{g_r}   K~_r = k_r e^{g_r}   K^_r = k_r e^{g_{L-1} - g_r}
//   A_{ri} = beta_r <k_r e^{g_r - g_m}, k_i e^{g_m - g_i}>   (i < r)
//   P_{ri} =        <q_r e^{g_r - g_m}, k_i e^{g_m - g_i}>   (i <= r)
//   T = (I + A)^{-1},  W = T diag(beta) K~,  U0 = T diag(beta) V
//   U = U0 - W S,  O = dk^{-1/2} (Q~ S + P U),  S' = Diag(e^{g_{L-1}}) S + K^^T U
//
// g_m is the value at the middle token of the chunk; splitting the decay of
// A and P there halves the largest exponent that is formed (products are
// unchanged).  T is formed by forward substitution, one column per thread.
#include "kda_common.cuh"
#include "kda_launch.h"
#include "ptx.cuh"

namespace kda {
namespace {

// ---------------------------------------------------------------- K0 ------
__global__ void __launch_bounds__(1024)
chunk_prep_kernel(WsHeader* hdr, int32_t* chunk_offsets, const int32_t* __restrict__ cu,
                  int N, int T, int fixed_num_chunks)
{
    __shared__ int warp_sums[32];
    __shared__ int s_carry, s_bad;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (cu == nullptr) {
        if (tid == 0) { hdr->status = kStatusOk; hdr->num_chunks = fixed_num_chunks; hdr->runtime_err = 0; hdr->next_pair = 0; }
        return;
    }
    if (tid == 0) { s_carry = 0; s_bad = (cu[0] != 0 || cu[N] != T) ? 1 : 0; }
    __syncthreads();
    for (int base = 0; base < N; base += 1024) {
        const int s = base + tid;
        int cnt = 0;
        if (s < N) {
            const int len = cu[s + 1] - cu[s];
            if (len < 0) atomicOr(&s_bad, 1);
            cnt = len > 0 ? (len + kChunk - 1) / kChunk : 0;
        }
        int incl = cnt;  // inclusive warp scan
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        if (lane == 31) warp_sums[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int w = warp_sums[lane];
            int wi = w;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, wi, off);
                if (lane >= off) wi += y;
            }
            warp_sums[lane] = wi - w;  // exclusive prefix of warp totals
        }
        __syncthreads();
        const int excl = s_carry + warp_sums[warp] + incl - cnt;
        if (s < N) chunk_offsets[s] = excl;
        __syncthreads();
        if (tid == 1023) s_carry = excl + cnt;
        __syncthreads();
    }
    if (tid == 0) {
        chunk_offsets[N] = s_carry;
        const bool bad = s_bad != 0;
        hdr->status = bad ? kStatusBadSeqlens : kStatusOk;
        hdr->num_chunks = bad ? 0 : s_carry;
        hdr->runtime_err = 0;
        hdr->next_pair = 0;
    }
}

template <int DK, int DV>
using SimtRec = F32Rec<DK, DV>;

// ---------------------------------------------------------------- K1 ------
template <typename T, int DK, int DV>
struct IntraSmem {
    static constexpr int LDK = DK + 4;   // padded row strides (float4-aligned)
    static constexpr int LDN = (DK > DV ? DK : DV) + 4;
    static constexpr int LDA = kChunk + 1;
    float g[kChunk][DK];
    float bufA[kChunk][LDK];   // K~ with mid reference, later K~ (chunk-start reference)
    float bufB[kChunk][LDK];   // K- (k e^{g_m - g})
    float bufC[kChunk][LDN];   // Q~ with mid reference, later V
    float Am[kChunk][LDA];     // A, later T diag(beta)
    float Pm[kChunk][LDA];
    float beta[kChunk];
    float gref[DK], gend[DK];
};

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(256)
intra_chunk_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                        const float* __restrict__ log_alpha, const float* __restrict__ beta,
                        ChunkMap map, const WsHeader* __restrict__ hdr, float* __restrict__ records,
                        float* __restrict__ tmat, int H, size_t max_chunks, int gate)
{
    using R = SimtRec<DK, DV>;
    using Sm = IntraSmem<T, DK, DV>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Sm& sm = *reinterpret_cast<Sm*>(smem_raw);

    if (hdr->status != kStatusOk) return;
    const int c = blockIdx.x, h = blockIdx.y;
    if (c >= hdr->num_chunks) return;
    int s, tok0, L;
    map.locate(c, s, tok0, L);
    float* rec = records + ((size_t)h * max_chunks + c) * R::FLOATS;
    const int tid = threadIdx.x;
    const size_t rowk = (size_t)H * DK, rowv = (size_t)H * DV;

    // a. in-chunk cumulative log-decay per key channel; padded rows add 0
    if (tid < DK) {
        // per-channel gate: [.., H, DK]; per-head gate: [.., H] (the same value
        // for every channel); no gate: log-decay 0
        const size_t rstride = gate == kGateChannel ? rowk : (size_t)H;
        const float* la = gate == kGateChannel ? log_alpha + (size_t)tok0 * rowk + (size_t)h * DK + tid
                                               : log_alpha + (size_t)tok0 * H + h;
        float acc = 0.f;
#pragma unroll 8
        for (int r = 0; r < kChunk; ++r) {
            acc += (r < L && gate != kGateNone) ? la[(size_t)r * rstride] : 0.f;
            sm.g[r][tid] = acc;
        }
    } else if (tid >= 128 && tid < 128 + kChunk) {
        const int r = tid - 128;
        sm.beta[r] = (r < L) ? beta[(size_t)(tok0 + r) * H + h] : 0.f;
    }
    __syncthreads();
    bool wide = false;
    if (tid < DK) {
        sm.gref[tid] = sm.g[(L - 1) >> 1][tid];
        sm.gend[tid] = sm.g[L - 1][tid];
        wide = fmaxf(sm.g[0][tid] - sm.gref[tid], sm.gref[tid] - sm.gend[tid]) > 60.f;
    }
    // Strong decay: the split factors e^{+-(g - g_m)} could overflow, so this
    // chunk forms A and P exactly (every exponent <= 0) from the raw k and q.
    const bool strong = __syncthreads_or(wide);

    // b. decayed operands; Q~ and K^ go straight to the record
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
            const float em = expf(gg - sm.gref[ch]);
            sm.bufA[r][ch] = kk * em;
            sm.bufB[r][ch] = kk * expf(sm.gref[ch] - gg);
            sm.bufC[r][ch] = qq * em;
        } else {
            sm.bufA[r][ch] = kk;
            sm.bufC[r][ch] = qq;
        }
        rec[R::QT + (size_t)r * DK + ch] = qq * expf(gg);
        rec[R::KH + (size_t)r * DK + ch] = kk * expf(sm.gend[ch] - gg);
    }
    __syncthreads();

    // c. A (strictly lower, beta-weighted) and P (lower incl. diagonal)
    if (strong) {   // exact: one warp per (r, i), lanes over channels
        const int warp = tid >> 5, lane = tid & 31;
        for (int pr = warp; pr < kChunk * kChunk; pr += 8) {
            const int r = pr >> 6, i = pr & 63;
            float sa = 0.f, sp = 0.f;
            if (i <= r) {
                for (int c = lane; c < DK; c += 32) {
                    const float w = expf(sm.g[r][c] - sm.g[i][c]);
                    sa += sm.bufA[r][c] * sm.bufA[i][c] * w;
                    sp += sm.bufC[r][c] * sm.bufA[i][c] * w;
                }
#pragma unroll
                for (int off = 16; off; off >>= 1) {
                    sa += __shfl_xor_sync(0xffffffffu, sa, off);
                    sp += __shfl_xor_sync(0xffffffffu, sp, off);
                }
            }
            if (lane == 0) {
                sm.Am[r][i] = (i < r) ? sm.beta[r] * sa : 0.f;
                sm.Pm[r][i] = (i <= r) ? sp : 0.f;
            }
        }
    } else {
        const int ty = tid >> 4, tx = tid & 15;
        float acc_a[4][4], acc_p[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) { acc_a[a][b] = 0.f; acc_p[a][b] = 0.f; }
        for (int ch = 0; ch < DK; ch += 4) {
            float4 kr[4], qr[4], kc[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                kr[a] = *reinterpret_cast<const float4*>(&sm.bufA[ty + 16 * a][ch]);
                qr[a] = *reinterpret_cast<const float4*>(&sm.bufC[ty + 16 * a][ch]);
                kc[a] = *reinterpret_cast<const float4*>(&sm.bufB[tx + 16 * a][ch]);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    acc_a[a][b] += kr[a].x * kc[b].x + kr[a].y * kc[b].y + kr[a].z * kc[b].z + kr[a].w * kc[b].w;
                    acc_p[a][b] += qr[a].x * kc[b].x + qr[a].y * kc[b].y + qr[a].z * kc[b].z + qr[a].w * kc[b].w;
                }
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int r = ty + 16 * a, i = tx + 16 * b;
                sm.Am[r][i] = (i < r) ? sm.beta[r] * acc_a[a][b] : 0.f;
                sm.Pm[r][i] = (i <= r) ? acc_p[a][b] : 0.f;
            }
    }  // !strong
    __syncthreads();

    // d. T = (I + A)^{-1} by forward substitution (threads 0..63, one column
    //    each); meanwhile the other threads stage K~ (chunk-start reference)
    //    and V for the W / U0 products.
    float x[kChunk];
    if (tid < kChunk) {
#pragma unroll
        for (int r = 0; r < kChunk; ++r) {
            float a0 = (r == tid) ? 1.f : 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
            for (int i = 0; i + 3 < r; i += 4) {
                a0 -= sm.Am[r][i] * x[i];
                a1 -= sm.Am[r][i + 1] * x[i + 1];
                a2 -= sm.Am[r][i + 2] * x[i + 2];
                a3 -= sm.Am[r][i + 3] * x[i + 3];
            }
#pragma unroll
            for (int i = r & ~3; i < r; ++i) a0 -= sm.Am[r][i] * x[i];
            x[r] = (a0 + a1) + (a2 + a3);
        }
        if (tmat) {   // T itself, for the backward pass
            float* tm = tmat + ((size_t)h * max_chunks + c) * kChunk * kChunk;
#pragma unroll
            for (int r = 0; r < kChunk; ++r) tm[r * kChunk + tid] = x[r];
        }
    } else {
        for (int idx = tid - kChunk; idx < kChunk * DK; idx += 256 - kChunk) {
            const int r = idx / DK, ch = idx - r * DK;
            float kk = 0.f;
            if (r < L) kk = to_f32(k[(size_t)(tok0 + r) * rowk + (size_t)h * DK + ch]);
            sm.bufA[r][ch] = kk * expf(sm.g[r][ch]);
        }
        for (int idx = tid - kChunk; idx < kChunk * DV; idx += 256 - kChunk) {
            const int r = idx / DV, ch = idx - r * DV;
            sm.bufC[r][ch] = (r < L) ? to_f32(v[(size_t)(tok0 + r) * rowv + (size_t)h * DV + ch]) : 0.f;
        }
    }
    __syncthreads();
    if (tid < kChunk) {
        const float bt = sm.beta[tid];
#pragma unroll
        for (int r = 0; r < kChunk; ++r) sm.Am[r][tid] = x[r] * bt;  // T diag(beta)
    }
    __syncthreads();

    // e. W = T diag(beta) K~ and U0 = T diag(beta) V (columns [0,DK) | [DK,DK+DV))
    {
        constexpr int NCOL = (DK + DV) / 16;
        const int ty = tid >> 4, tx = tid & 15;
        float acc[4][NCOL];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < NCOL; ++b) acc[a][b] = 0.f;
        for (int i = 0; i < kChunk; ++i) {
            float t[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) t[a] = sm.Am[ty + 16 * a][i];
#pragma unroll
            for (int b = 0; b < NCOL; ++b) {
                const int n = tx + 16 * b;
                const float y = (n < DK) ? sm.bufA[i][n] : sm.bufC[i][n - DK];
#pragma unroll
                for (int a = 0; a < 4; ++a) acc[a][b] = fmaf(t[a], y, acc[a][b]);
            }
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < NCOL; ++b) {
                const int r = ty + 16 * a, n = tx + 16 * b;
                if (n < DK) rec[R::W + (size_t)r * DK + n] = acc[a][b];
                else rec[R::U0 + (size_t)r * DV + (n - DK)] = acc[a][b];
            }
    }

    // f. P and the chunk's total decay
    for (int idx = tid; idx < kChunk * kChunk; idx += 256)
        rec[R::P + idx] = sm.Pm[idx >> 6][idx & 63];
    if (tid < DK) rec[R::GC + tid] = expf(sm.gend[tid]);
}

// ---------------------------------------------------------------- K2 ------
constexpr int kSlice = 64;  // value columns per inter-chunk CTA
constexpr int kInterThreads = 256;

// Shared memory of K2.  The record tiles are unpadded copies of the record
// rows: every access below is a warp broadcast or along consecutive columns.
template <int DK>
struct InterSmem {
    float S[DK][kSlice + 1];
    float W[kChunk][DK];
    float Qt[kChunk][DK];
    float Kh[kChunk][DK];
    float P[kChunk][kChunk];
    float U0[kChunk][kSlice];
    float U[kChunk][kSlice + 4];
    float gC[DK];
};

// One CTA (8 warps) per (sequence, head, 64-wide value slice), serial over the
// chunks.  The loads of chunk n+1 are software-pipelined with the work of
// chunk n: W, Q~ and the U0 slice are fetched (cp.async) once step 1 of chunk n
// is done with them, P, K^ and gamma once steps 2 and 3 are.
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kInterThreads, 1)
inter_chunk_simt_kernel(const float* __restrict__ initial_state, float* __restrict__ final_state,
                        T* __restrict__ o, float* __restrict__ states, ChunkMap map,
                        const WsHeader* __restrict__ hdr, const float* __restrict__ records, int H,
                        size_t max_chunks, float scale)
{
    using R = SimtRec<DK, DV>;
    using Sm = InterSmem<DK>;
    constexpr int NT = kInterThreads;
    constexpr int CPT = kSlice * DK / NT;   // step-3 columns per thread
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Sm& sm = *reinterpret_cast<Sm*>(smem_raw);

    if (hdr->status != kStatusOk) return;
    const int s = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * kSlice;
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    const size_t state_off = ((size_t)s * H + h) * DK * DV;

    for (int idx = tid; idx < DK * kSlice; idx += NT) {
        const int r = idx / kSlice, j = idx - r * kSlice;
        sm.S[r][j] = initial_state ? initial_state[state_off + (size_t)r * DV + j0 + j] : 0.f;
    }

    const int first = map.seq_first_chunk(s);
    const int nch = map.seq_num_chunks(s);
    const int tok_begin = map.seq_token_begin(s), tok_end = map.seq_token_end(s);

    auto issue_a = [&](int n) {   // W, Q~, U0 slice of chunk n
        const float* rec = records + ((size_t)h * max_chunks + first + n) * R::FLOATS;
        for (int e = tid; e < kChunk * DK / 4; e += NT) {
            ptx::cp_async16(&sm.W[0][0] + 4 * e, rec + R::W + 4 * e);
            ptx::cp_async16(&sm.Qt[0][0] + 4 * e, rec + R::QT + 4 * e);
        }
        for (int e = tid; e < kChunk * kSlice / 4; e += NT) {
            const int r = e / (kSlice / 4), c4 = (e - r * (kSlice / 4)) * 4;
            ptx::cp_async16(&sm.U0[r][c4], rec + R::U0 + (size_t)r * DV + j0 + c4);
        }
    };
    auto issue_b = [&](int n) {   // P, K^, gamma of chunk n
        const float* rec = records + ((size_t)h * max_chunks + first + n) * R::FLOATS;
        for (int e = tid; e < kChunk * DK / 4; e += NT) ptx::cp_async16(&sm.Kh[0][0] + 4 * e, rec + R::KH + 4 * e);
        for (int e = tid; e < kChunk * kChunk / 4; e += NT) ptx::cp_async16(&sm.P[0][0] + 4 * e, rec + R::P + 4 * e);
        for (int e = tid; e < DK / 4; e += NT) ptx::cp_async16(&sm.gC[0] + 4 * e, rec + R::GC + 4 * e);
    };

    if (nch > 0) {
        issue_a(0);
        ptx::cp_async_commit();
        issue_b(0);
        ptx::cp_async_commit();
    }
    for (int n = 0; n < nch; ++n) {
        ptx::cp_async_wait<1>();   // this thread's part of W, Q~, U0 of chunk n has landed
        __syncthreads();           // everyone's; S of the previous chunk is complete
        if (states) {   // the state entering this chunk, for the backward pass
            float* st = states + ((size_t)h * max_chunks + first + n) * DK * DV;
            for (int idx = tid; idx < DK * kSlice; idx += NT) {
                const int r = idx / kSlice, j = idx - r * kSlice;
                st[(size_t)r * DV + j0 + j] = sm.S[r][j];
            }
        }

        // 1. W S and Q~ S for rows r = wp + 8a, columns lane and lane + 32
        float ws[8][2], qs[8][2];
#pragma unroll
        for (int a = 0; a < 8; ++a) { ws[a][0] = ws[a][1] = qs[a][0] = qs[a][1] = 0.f; }
        for (int c = 0; c < DK; c += 4) {
            float s0[4], s1[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) { s0[t] = sm.S[c + t][lane]; s1[t] = sm.S[c + t][lane + 32]; }
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const float4 w = *reinterpret_cast<const float4*>(&sm.W[wp + 8 * a][c]);
                const float4 qv = *reinterpret_cast<const float4*>(&sm.Qt[wp + 8 * a][c]);
                ws[a][0] += w.x * s0[0] + w.y * s0[1] + w.z * s0[2] + w.w * s0[3];
                ws[a][1] += w.x * s1[0] + w.y * s1[1] + w.z * s1[2] + w.w * s1[3];
                qs[a][0] += qv.x * s0[0] + qv.y * s0[1] + qv.z * s0[2] + qv.w * s0[3];
                qs[a][1] += qv.x * s1[0] + qv.y * s1[1] + qv.z * s1[2] + qv.w * s1[3];
            }
        }
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            const int r = wp + 8 * a;
            sm.U[r][lane] = sm.U0[r][lane] - ws[a][0];
            sm.U[r][lane + 32] = sm.U0[r][lane + 32] - ws[a][1];
        }
        __syncthreads();   // W, Q~, U0 are free; U is complete
        if (n + 1 < nch) {
            issue_a(n + 1);
            ptx::cp_async_commit();
            ptx::cp_async_wait<1>();   // P, K^, gamma of chunk n have landed
        } else {
            ptx::cp_async_wait<0>();
        }
        __syncthreads();

        // 2. O = scale (Q~ S + P U)
        if (o) {
            for (int i = 0; i < kChunk; i += 4) {
                float u0[4], u1[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) { u0[t] = sm.U[i + t][lane]; u1[t] = sm.U[i + t][lane + 32]; }
#pragma unroll
                for (int a = 0; a < 8; ++a) {
                    const float4 p = *reinterpret_cast<const float4*>(&sm.P[wp + 8 * a][i]);
                    qs[a][0] += p.x * u0[0] + p.y * u0[1] + p.z * u0[2] + p.w * u0[3];
                    qs[a][1] += p.x * u1[0] + p.y * u1[1] + p.z * u1[2] + p.w * u1[3];
                }
            }
            const int chunk_tok0 = tok_begin + n * kChunk;
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const int tok = chunk_tok0 + wp + 8 * a;
                if (tok < tok_end) {
                    T* orow = o + ((size_t)tok * H + h) * DV + j0;
                    orow[lane] = from_f32<T>(scale * qs[a][0]);
                    orow[lane + 32] = from_f32<T>(scale * qs[a][1]);
                }
            }
        }

        // 3. S' = Diag(gC) S + K^^T U: key row c, CPT columns from jb
        {
            const int c = tid % DK, jb = (tid / DK) * CPT;
            float acc[CPT];
            const float gc = sm.gC[c];
#pragma unroll
            for (int j = 0; j < CPT; ++j) acc[j] = gc * sm.S[c][jb + j];
            for (int r = 0; r < kChunk; ++r) {
                const float kh = sm.Kh[r][c];
#pragma unroll
                for (int j = 0; j < CPT; j += 4) {
                    const float4 u = *reinterpret_cast<const float4*>(&sm.U[r][jb + j]);
                    acc[j] += kh * u.x; acc[j + 1] += kh * u.y;
                    acc[j + 2] += kh * u.z; acc[j + 3] += kh * u.w;
                }
            }
#pragma unroll
            for (int j = 0; j < CPT; ++j) sm.S[c][jb + j] = acc[j];   // this thread's own segment
        }
        __syncthreads();   // P, K^, gamma are free
        if (n + 1 < nch) {
            issue_b(n + 1);
            ptx::cp_async_commit();
        }
    }
    __syncthreads();
    if (final_state) {
        for (int idx = tid; idx < DK * kSlice; idx += NT) {
            const int r = idx / kSlice, j = idx - r * kSlice;
            final_state[state_off + (size_t)r * DV + j0 + j] = sm.S[r][j];
        }
    }
}

template <typename T, int DK, int DV>
cudaError_t launch_intra_t(const ChunkArgs& a) {
    if (a.max_chunks == 0) return cudaSuccess;
    ChunkMap map{a.cu_seqlens, a.chunk_offsets, a.num_seqs, a.T, a.fixed_chunks_per_seq};
    auto k1 = intra_chunk_simt_kernel<T, DK, DV>;
    const int smem = (int)sizeof(IntraSmem<T, DK, DV>);
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)a.max_chunks, (unsigned)a.H);
    k1<<<grid, 256, smem, a.stream>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v),
        a.log_alpha, a.beta, map, static_cast<const WsHeader*>(a.ws_header),
        static_cast<float*>(a.records), a.tmat, a.H, a.max_chunks, a.gate);
    return cudaGetLastError();
}

template <typename T, int DK, int DV>
cudaError_t launch_inter_t(const ChunkArgs& a) {
    ChunkMap map{a.cu_seqlens, a.chunk_offsets, a.num_seqs, a.T, a.fixed_chunks_per_seq};
    auto k2 = inter_chunk_simt_kernel<T, DK, DV>;
    const int smem = (int)sizeof(InterSmem<DK>);
    cudaError_t e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)a.num_seqs, (unsigned)a.H, (unsigned)(DV / kSlice));
    k2<<<grid, kInterThreads, smem, a.stream>>>(a.initial_state, a.final_state, static_cast<T*>(a.o), a.states, map,
                                       static_cast<const WsHeader*>(a.ws_header),
                                       static_cast<const float*>(a.records), a.H, a.max_chunks,
                                       a.scale);
    return cudaGetLastError();
}

#define KDA_DISPATCH(FN, a)                                                         \
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

size_t simt_record_bytes(int dk, int dv) {
    if (dk == 128 && dv == 128) return SimtRec<128, 128>::FLOATS * sizeof(float);
    if (dk == 128 && dv == 64) return SimtRec<128, 64>::FLOATS * sizeof(float);
    if (dk == 64 && dv == 128) return SimtRec<64, 128>::FLOATS * sizeof(float);
    if (dk == 64 && dv == 64) return SimtRec<64, 64>::FLOATS * sizeof(float);
    return 0;
}

cudaError_t launch_chunk_prep(const ChunkArgs& a) {
    const int fixed_chunks = a.cu_seqlens ? 0 : a.num_seqs * a.fixed_chunks_per_seq;
    chunk_prep_kernel<<<1, 1024, 0, a.stream>>>(static_cast<WsHeader*>(a.ws_header), a.chunk_offsets,
                                               a.cu_seqlens, a.num_seqs, a.T, fixed_chunks);
    return cudaGetLastError();
}

cudaError_t launch_chunk_intra(const ChunkArgs& a) { KDA_DISPATCH(launch_intra_t, a); }

cudaError_t launch_chunk_inter(const ChunkArgs& a) {
    if (a.num_seqs == 0) return cudaSuccess;
    KDA_DISPATCH(launch_inter_t, a);
}

}  // namespace kda
