// kda_inter_tc.cu -- the forward inter-chunk kernel on the sm_100a tensor cores
// (bf16 inputs): the chunk-to-chunk state recurrence, with the value dimension
// split into slices of NS columns (NS = 32, 64 or 128, chosen per call).
//
// The state is carried between chunks (the chunk-wise scheme of the
// kongchang.com page, section "硬件效率的优化策略"); with the records of the
// intra-chunk kernel, per chunk and value slice (the algebra of the daiw.net
// update equation, section "KDA 的更新式", unrolled over a chunk):
//
//   U = U0 - W S,   O = d_k^{-1/2} (Q~ S + P U),   S <- Diag(gamma_C) S + K^^T U
//
// One CTA (8 warps) per (sequence, head, value slice), serial over the
// sequence's chunks; packed sequences are started longest first.  The fp32 state slice is resident in TMEM for the whole
// sequence; its fp16 copy in shared memory is the B operand of [W; Q~] S.
// Records arrive by bulk copy into a double buffer.  Per chunk: MMA3 [W; Q~] S
// -> R3, U = U0 - W S (fp16), then MMA4 [*; P] U onto R3 and MMA5 K^^T U onto
// the state; the output rows of a chunk are written during the next chunk's
// MMA3 (R3 is double-buffered).
//
// The slice width trades the length of the serial chain against the work per
// CTA: narrow slices (32 columns) put more CTAs on a long sequence and shorten
// each chunk's conversions; wide slices (128 columns) read each record once
// instead of once per slice when there are enough (sequence, head) pairs to
// fill the GPU.
//
// Every thread polls the mbarriers (one CTA per SM: there is no co-resident
// CTA to give issue slots to, and the chain is latency-bound); a CTA whose wait
// gives up records KDA_ERR_TIMEOUT, drains the copies and MMAs it issued and
// returns.
#include <cuda_fp16.h>

#include "kda_common.cuh"
#include "kda_launch.h"
#include "kda_tc_common.cuh"
#include "ptx.cuh"

namespace kda {
namespace {

using namespace ptx;

template <int DK, int DV, int NS>
struct K2fSmem {
    using R = TcRec<DK, DV>;
    static constexpr int NT = NS > 64 ? NS / 64 : 1;        // 64-column tiles of a slice
    // one stage: [WQ][KH][P][U0 tiles][GC]; P directly after KH, so the 128-row
    // A operand [*; P] reads the tail of KH as its (unused) rows 0..63
    static constexpr uint32_t WQ = 0;
    static constexpr uint32_t KH = WQ + R::WQ_BYTES;
    static constexpr uint32_t P = KH + R::KH_BYTES;
    static constexpr uint32_t U0 = P + 8192;
    static constexpr uint32_t GC = U0 + NT * 8192;
    static constexpr uint32_t STAGE = (GC + DK * 4 + 1023) / 1024 * 1024;
    static constexpr uint32_t S16 = 2 * STAGE;              // fp16 state slice: NT tiles of 128 rows x 128 B
    static constexpr uint32_t U16 = S16 + NT * 16384;       // fp16 U: NT tiles of 64 rows x 128 B
    static constexpr uint32_t END = U16 + NT * 8192;
    static constexpr uint32_t TX_BYTES = R::WQ_BYTES + R::KH_BYTES + 8192 + NT * 8192 + DK * 4;
    static constexpr uint32_t TMEM_COLS = 3 * NS <= 128 ? 128 : (3 * NS <= 256 ? 256 : 512);
    static_assert(END + 1024 <= 232448, "shared memory");
};

// N consecutive TMEM columns of this thread's lane (N = 16, 32 or 64), waited for.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float* v) {
    if constexpr (N == 16) {
        float t[16];
        tmem_ld16(taddr, t);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = t[i];
    } else {
#pragma unroll
        for (int c = 0; c < N; c += 32) {
            float t[32];
            tmem_ld32_sync(taddr + c, t);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[c + i] = t[i];
        }
    }
}
template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const float* v) {
    if constexpr (N == 16) {
        float t[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) t[i] = v[i];
        tmem_st16(taddr, t);
        tmem_wait_st();
    } else {
#pragma unroll
        for (int c = 0; c < N; c += 32) {
            float t[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) t[i] = v[c + i];
            tmem_st32_sync(taddr + c, t);
        }
    }
}

template <int DK, int DV, int NS>
__global__ void __launch_bounds__(256, 1)
inter_chunk_fwd_tc_kernel(const float* __restrict__ initial_state, float* __restrict__ final_state,
                          __nv_bfloat16* __restrict__ o, ChunkMap map, WsHeader* hdr,
                          const unsigned char* __restrict__ records, int H, size_t max_chunks, float scale,
                          const int* __restrict__ seq_order, float* __restrict__ states)
{
    using Sm = K2fSmem<DK, DV, NS>;
    using R = TcRec<DK, DV>;
    constexpr int CPT = NS / 2;          // columns per thread: the two warpgroups split a slice
    constexpr int NT = Sm::NT;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar_full[2], bar_mma;
    __shared__ uint32_t s_tmem;

    if (hdr->status != kStatusOk) return;
    // CTAs are started in blockIdx order: all slices of one (sequence, head)
    // pair, pairs sequence by sequence, sequences longest first (seq_order)
    constexpr int NZ = DV / NS;
    const int pair = (int)blockIdx.x / NZ, si = pair / H;
    const int s = seq_order ? seq_order[si] : si, h = pair - si * H, j0 = ((int)blockIdx.x - pair * NZ) * NS;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int lane_row = (warp & 3) * 32 + (tid & 31);   // TMEM lane = MMA row
    const int wg = warp >> 2;                            // warpgroup: columns [CPT wg, CPT wg + CPT)
    const int first = map.seq_first_chunk(s), nch = map.seq_num_chunks(s);
    const int tok_begin = map.seq_token_begin(s), tok_end = map.seq_token_end(s);
    const size_t state_off = ((size_t)s * H + h) * DK * DV;
    const int u0_tile = j0 >> 6, u0_col = j0 & 63;        // where the slice sits in the record's U0 tiles

    if (tid == 0) {
        mbar_init(&bar_full[0], 1);
        mbar_init(&bar_full[1], 1);
        mbar_init(&bar_mma, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&s_tmem, Sm::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    // [W S; Q~ S + P U] of chunk n at columns NS (n & 1) (128 lanes x NS), then the state slice
    auto r3 = [&](int n) -> uint32_t { return tmem + (uint32_t)(NS * (n & 1)); };
    const uint32_t SACC = tmem + 2 * NS;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t cb = (uint32_t)(CPT * wg);             // this thread's first column in the slice
    float range_max = 0.f;

    auto issue = [&](int n) {   // bulk-copy chunk n's records into stage n & 1
        if (n >= nch) return;
        unsigned char* st = sm + (n & 1) * Sm::STAGE;
        const unsigned char* rec = records + ((size_t)h * max_chunks + first + n) * R::BYTES;
        uint64_t* bar = &bar_full[n & 1];
        mbar_arrive_expect_tx(bar, Sm::TX_BYTES);
        bulk_load(st + Sm::WQ, rec + R::WQ, R::WQ_BYTES, bar);
        bulk_load(st + Sm::KH, rec + R::KH, R::KH_BYTES, bar);
        bulk_load(st + Sm::P, rec + R::P, 8192, bar);
        bulk_load(st + Sm::U0, rec + R::U0 + u0_tile * 8192, NT * 8192, bar);
        bulk_load(st + Sm::GC, rec + R::GC, DK * 4, bar);
    };
    // fp16 copy of this thread's CPT state columns (row = key channel) into S16
    auto put_s16 = [&](const float* v) {
#pragma unroll
        for (int i8 = 0; i8 < CPT / 8; ++i8) {
            const uint32_t col = cb + 8 * i8;
            __align__(16) __half2 hv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a = v[8 * i8 + 2 * e], b = v[8 * i8 + 2 * e + 1];
                range_max = fmaxf(range_max, fmaxf(fabsf(a), fabsf(b)));
                hv[e] = __floats2half2_rn(a, b);
            }
            *reinterpret_cast<uint4*>(sm + Sm::S16 + (col >> 6) * 16384 + sw128_offset(lane_row, (col & 63) * 2)) =
                *reinterpret_cast<const uint4*>(hv);
        }
    };
    // output rows (lanes 64..127) of chunk n from R3[n & 1]: warps 2, 3, 6, 7
    auto write_o = [&](int n) {
        const int r = lane_row - 64;
        const int tok = tok_begin + n * kChunk + r;
        float v[CPT];
        tmem_ld_cols<CPT>(r3(n) + lane_base + cb, v);
        if (o && tok < tok_end) {
            __nv_bfloat16* dst = o + ((size_t)tok * H + h) * DV + j0 + cb;
#pragma unroll
            for (int i8 = 0; i8 < CPT / 8; ++i8) {
                __align__(16) __nv_bfloat162 bv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    bv[e] = __floats2bfloat162_rn(scale * v[8 * i8 + 2 * e], scale * v[8 * i8 + 2 * e + 1]);
                *reinterpret_cast<uint4*>(dst + 8 * i8) = *reinterpret_cast<const uint4*>(bv);
            }
        }
    };

    // initial state slice -> TMEM accumulator and fp16 operand copy
    if (lane_row < DK) {
        float v[CPT];
#pragma unroll
        for (int i = 0; i < CPT; i += 4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (initial_state)
                x = *reinterpret_cast<const float4*>(initial_state + state_off + (size_t)lane_row * DV + j0 + cb + i);
            v[i] = x.x; v[i + 1] = x.y; v[i + 2] = x.z; v[i + 3] = x.w;
        }
        tmem_st_cols<CPT>(SACC + lane_base + cb, v);
        put_s16(v);
    }
    if (tid == 0) {
        issue(0);
        issue(1);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    bool aborted = false;
    uint32_t mma_phase = 0;
    int mma_pending = 0;   // a commit on bar_mma not yet waited for
    // chunk j's records land on bar_full[j & 1] (phase parity (j >> 1) & 1);
    // chunks copies_done .. copies_issued - 1 are in flight (drained on abort)
    int copies_issued = nch < 2 ? nch : 2, copies_done = 0;
    int n = 0;
    for (; n < nch; ++n) {
        const int b = n & 1;
        unsigned char* st = sm + b * Sm::STAGE;
        bool ok = mbar_wait_cycles(&bar_full[b], (n >> 1) & 1, kWaitCycles);
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        copies_done = n + 1;

        const uint32_t R3 = r3(n);
        // MMA3: [W; Q~] S -> R3
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc = instr_desc(kFmtF16, 128, NS, false, true);
            const uint32_t a0 = smem_u32(st + Sm::WQ), b0 = smem_u32(sm + Sm::S16);
#pragma unroll
            for (int kb = 0; kb < DK / 64; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(R3, smem_desc(a0 + kb * 16384 + ks * 32, 16, 1024, kLayoutSW128),
                            smem_desc(b0 + kb * 8192 + ks * 2048, 16384, 1024, kLayoutSW128), idesc,
                            (kb | ks) != 0);
            mma_commit(&bar_mma);
        }
        mma_pending = 1;
        // meanwhile: S_acc <- Diag(gC) S_acc (MMA3 reads the fp16 copy, not S_acc),
        // and the previous chunk's output rows; backward mode: the state entering
        // this chunk
        if (lane_row < DK) {
            const float gc = reinterpret_cast<const float*>(st + Sm::GC)[lane_row];
            float v[CPT];
            tmem_ld_cols<CPT>(SACC + lane_base + cb, v);
            if (states) {
                float* dst = states + (((size_t)h * max_chunks + first + n) * DK + lane_row) * DV + j0 + cb;
#pragma unroll
                for (int i = 0; i < CPT; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
            }
#pragma unroll
            for (int i = 0; i < CPT; ++i) v[i] *= gc;
            tmem_st_cols<CPT>(SACC + lane_base + cb, v);
        }
        if (n > 0 && lane_row >= 64) write_o(n - 1);
        ok = mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        mma_phase ^= 1;
        mma_pending = 0;
        tc_fence_after();

        // U = U0 - W S  (rows 0..63 = tokens), fp16 -> U16
        if (lane_row < 64) {
            const int r = lane_row;
            float v[CPT];
            tmem_ld_cols<CPT>(R3 + lane_base + cb, v);
#pragma unroll
            for (int i8 = 0; i8 < CPT / 8; ++i8) {
                const uint32_t col = cb + 8 * i8;                  // column within the slice
                const uint32_t ucol = u0_col + col;                // column within the record's U0 tiles
                const uint4 u0raw = *reinterpret_cast<const uint4*>(st + Sm::U0 + (ucol >> 6) * 8192 + sw128_offset(r, (ucol & 63) * 2));
                const __half2* u0 = reinterpret_cast<const __half2*>(&u0raw);
                __align__(16) __half2 hv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 u0f = __half22float2(u0[e]);
                    const float ua = u0f.x - v[8 * i8 + 2 * e], ub = u0f.y - v[8 * i8 + 2 * e + 1];
                    range_max = fmaxf(range_max, fmaxf(fabsf(ua), fabsf(ub)));
                    hv[e] = __floats2half2_rn(ua, ub);
                }
                *reinterpret_cast<uint4*>(sm + Sm::U16 + (col >> 6) * 8192 + sw128_offset(r, (col & 63) * 2)) =
                    *reinterpret_cast<const uint4*>(hv);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // MMA4: [*; P] U += R3 ; MMA5: K^^T U += S_acc
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc = instr_desc(kFmtF16, 128, NS, false, true);
            constexpr uint32_t idesc_t = instr_desc(kFmtF16, 128, NS, true, true);
            const uint32_t pa = smem_u32(st + Sm::P) - 8192, ub = smem_u32(sm + Sm::U16);
            const uint32_t ka = smem_u32(st + Sm::KH);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_f16(R3, smem_desc(pa + ks * 32, 16, 1024, kLayoutSW128),
                        smem_desc(ub + ks * 2048, 8192, 1024, kLayoutSW128), idesc, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_f16(SACC, smem_desc(ka + ks * 2048, 8192, 1024, kLayoutSW128),
                        smem_desc(ub + ks * 2048, 8192, 1024, kLayoutSW128), idesc_t, true);
            mma_commit(&bar_mma);
        }
        mma_pending = 1;
        ok = mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        mma_phase ^= 1;
        mma_pending = 0;
        tc_fence_after();
        if (tid == 0) {
            fence_proxy_async_smem();
            issue(n + 2);   // this stage is no longer read
        }
        if (n + 2 < nch) copies_issued = n + 3;
        // next state's fp16 operand copy (the serial path); the output rows of
        // this chunk are written during the next chunk's MMA3
        if (lane_row < DK) {
            float v[CPT];
            tmem_ld_cols<CPT>(SACC + lane_base + cb, v);
            put_s16(v);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (aborted) {
        if (tid == 0) {
            flag_error(hdr, kStatusTimeout);
            // let MMAs and copies this CTA issued finish before its memory goes away
            if (mma_pending) (void)mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
            for (int j = copies_done; j < copies_issued; ++j)
                (void)mbar_wait_cycles(&bar_full[j & 1], (j >> 1) & 1, kWaitCycles / 8);
        }
    } else {
        if (nch > 0 && lane_row >= 64) write_o(nch - 1);
        if (final_state && lane_row < DK) {
            float v[CPT];
            tmem_ld_cols<CPT>(SACC + lane_base + cb, v);
            float* dst = final_state + state_off + (size_t)lane_row * DV + j0 + cb;
#pragma unroll
            for (int i = 0; i < CPT; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
    }
    if (range_max > kF16Limit) flag_error(hdr, kStatusRange);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, Sm::TMEM_COLS);
}

template <int DK, int DV, int NS>
cudaError_t launch_inter_fwd_tc_ns(const ChunkArgs& a) {
    ChunkMap map{a.cu_seqlens, a.chunk_offsets, a.num_seqs, a.T, a.fixed_chunks_per_seq};
    auto kern = inter_chunk_fwd_tc_kernel<DK, DV, NS>;
    const int smem = (int)K2fSmem<DK, DV, NS>::END + 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((size_t)a.num_seqs * a.H * (DV / NS));
    kern<<<grid, 256, smem, a.stream>>>(a.initial_state, a.final_state, static_cast<__nv_bfloat16*>(a.o), map,
                                        static_cast<WsHeader*>(a.ws_header),
                                        static_cast<const unsigned char*>(a.records), a.H, a.max_chunks, a.scale,
                                        a.seq_order, a.states);
    return cudaGetLastError();
}

// The slice width from the number of (sequence, head) chains: as narrow as
// keeps every chain's slices within one wave of CTAs (one per SM), as wide as
// the value dimension once the chains alone fill the GPU twice over.
template <int DK, int DV>
cudaError_t launch_inter_fwd_tc_t(const ChunkArgs& a) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long chains = (long long)a.num_seqs * a.H;
    if (chains * (DV / 32) <= sms) return launch_inter_fwd_tc_ns<DK, DV, 32>(a);
    if constexpr (DV == 128) {
        if (chains >= 2LL * sms) return launch_inter_fwd_tc_ns<DK, DV, 128>(a);
    }
    return launch_inter_fwd_tc_ns<DK, DV, 64>(a);
}

}  // namespace

cudaError_t launch_chunk_inter_fwd_tc(const ChunkArgs& a) {
    if (a.num_seqs == 0) return cudaSuccess;
    if (a.dk == 128 && a.dv == 128) return launch_inter_fwd_tc_t<128, 128>(a);
    if (a.dk == 128 && a.dv == 64) return launch_inter_fwd_tc_t<128, 64>(a);
    if (a.dk == 64 && a.dv == 128) return launch_inter_fwd_tc_t<64, 128>(a);
    if (a.dk == 64 && a.dv == 64) return launch_inter_fwd_tc_t<64, 64>(a);
    return cudaErrorInvalidValue;
}

}  // namespace kda
