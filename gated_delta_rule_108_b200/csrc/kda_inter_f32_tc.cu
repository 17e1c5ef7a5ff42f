// kda_inter_f32_tc.cu -- the forward inter-chunk kernel for fp32 inputs on the
// sm_100a tensor cores, products in split tf32 (hi.hi + hi.lo + lo.hi, fp32
// accumulation in tensor memory; see kda_intra_f32_tc.cu).
//
// The chunk-to-chunk state recurrence (the chunk-wise scheme of the
// kongchang.com page, section "硬件效率的优化策略"; the daiw.net update equation,
// section "KDA 的更新式", unrolled over a chunk), per chunk and value slice of
// NS = 32 or 64 columns, from the F32TcRec records of the fp32 tensor-core
// intra-chunk kernel:
//
//   MMA3  R3 = [W; Q~] S                 A [W; Q~] (hi | lo) in TMEM, B S^T in smem
//   U = U0 - W S                         fp32, on CUDA cores
//   MMA4  R3[64..127] += P U             A [*; P] in smem, B U^T in smem
//   MMA5  S <- Diag(gamma_C) S + K^^T U  A K^^T in TMEM, the state accumulated in TMEM
//   O = d_k^{-1/2} R3[64..127]
//
// tf32 operands are K-major, so the state and U are written transposed (one
// thread per TMEM lane, a warp's 32 lanes filling one 128-byte row).  The A
// operands of the next chunk come from global memory into registers while the
// current chunk's products run: [W; Q~] goes to TMEM once MMA3 has read the
// current one, K^^T once MMA5 has.  P, the U0 slice and gamma_C come by bulk
// copy into a double buffer.  U^T lives in the rows of the [*; P] tiles that
// MMA4 reads but does not use.
//
// One CTA (8 warps) per (sequence, head, value slice), serial over the
// sequence's chunks.  A chunk costs about the same at either slice width (the
// tensor core's time per instruction hardly depends on N at these sizes), so
// the launcher takes 64 columns when 32-column slices would need a second wave
// of CTAs.  With 64 columns (d_k = 128) tensor memory has room for one R3 only,
// and a chunk's output rows are read before the next chunk's MMA3.  Every wait is bounded; a CTA whose wait gives up records
// KDA_ERR_TIMEOUT, drains the copies and MMAs it issued and returns.
#include "kda_common.cuh"
#include "kda_launch.h"
#include "kda_tc_common.cuh"
#include "ptx.cuh"

namespace kda {
namespace {

using namespace ptx;

__device__ __forceinline__ void split_tf32_(float x, float& hi, float& lo) {
    hi = __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
    lo = x - hi;
}

template <int DK, int DV, int NS>
struct F32K2Smem {
    // one stage: P (2 tiles of 64 rows x 128 B, as in the record), the U0 slice
    // (NS/32 tiles of 64 rows x 128 B, as in the record), gamma_C
    static constexpr uint32_t SP = 0, SU0 = 16384, SGC = SU0 + (NS / 32) * 8192;
    static constexpr uint32_t STAGE = (SGC + DK * 4 + 1023) / 1024 * 1024;
    static constexpr uint32_t TX_BYTES = SGC + DK * 4;
    // [*; P] (hi | lo): 4 tiles (hi t0, hi t1, lo t0, lo t1) of 128 rows x 128 B,
    // P in rows 64..127.  Rows 0..63 (MMA4's unused rows) hold U^T (hi | lo):
    // tile (hl, t) = tokens 32t..32t+31, NS rows (value column) x 128 B
    static constexpr uint32_t PA = 2 * STAGE;
    static constexpr uint32_t UT_HALF = 2 * 16384;
    // S^T (hi | lo): DK/32 tiles of NS rows (value column) x 128 B each
    static constexpr uint32_t ST = PA + 4 * 16384;
    static constexpr uint32_t ST_TILE = NS * 128;
    static constexpr uint32_t ST_HALF = (DK / 32) * ST_TILE;
    static constexpr uint32_t END = ST + 2 * ST_HALF;
    static_assert(NS * 128 <= 8192, "U^T fits in the unused rows");
    static_assert(END + 1024 <= 232448, "shared memory");
};

template <int DK, int DV, int NS>
__global__ void __launch_bounds__(256, 1)
inter_chunk_f32_tc_kernel(const float* __restrict__ initial_state, float* __restrict__ final_state,
                          float* __restrict__ o, ChunkMap map, WsHeader* hdr, const float* __restrict__ records,
                          int H, size_t max_chunks, float scale)
{
    using Sm = F32K2Smem<DK, DV, NS>;
    using R = F32TcRec<DK, DV>;
    constexpr int NZ = DV / NS;
    constexpr int CPT = NS / 2;          // state / U / output columns per thread (two warpgroups)
    // R3 buffers: two (the output rows are written during the next chunk's MMA3)
    // when tensor memory has room
    constexpr int NB = (3 * NS + 2 * DK + 128 <= 512) ? 2 : 1;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar_full[2], bar_mma;
    __shared__ uint32_t s_tmem;

    if (hdr->status != kStatusOk) return;
    const int pair = (int)blockIdx.x / NZ, s = pair / H, h = pair - s * H;
    const int j0 = ((int)blockIdx.x - pair * NZ) * NS;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int lane_row = (warp & 3) * 32 + (tid & 31);   // TMEM lane
    const int wg = warp >> 2;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const int first = map.seq_first_chunk(s), nch = map.seq_num_chunks(s);
    const int tok_begin = map.seq_token_begin(s), tok_end = map.seq_token_end(s);
    const size_t state_off = ((size_t)s * H + h) * DK * DV;
    const bool chan = lane_row < DK;     // this lane holds a key channel of the state / K^^T

    if (tid == 0) {
        mbar_init(&bar_full[0], 1);
        mbar_init(&bar_full[1], 1);
        mbar_init(&bar_mma, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&s_tmem, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const uint32_t SACC = tmem;                                    // state slice: lanes = channel, NS columns
    auto r3 = [&](int n) -> uint32_t { return tmem + NS + NS * (uint32_t)(NB == 2 ? (n & 1) : 0); };   // 128 lanes x NS
    const uint32_t WQA = tmem + (1 + NB) * NS;                     // [W; Q~] hi at +0, lo at +DK
    const uint32_t KHA = WQA + 2 * DK;                             // K^^T hi at +0, lo at +64
    static_assert((1 + NB) * NS + 2 * DK + 128 <= 512, "tensor memory");
    const uint32_t cb = (uint32_t)(CPT * wg);                      // this thread's first column

    auto rec_of = [&](int n) { return records + ((size_t)h * max_chunks + first + n) * R::FLOATS; };
    auto issue = [&](int n) {   // P, the U0 slice and gamma_C of chunk n into stage n & 1
        if (n >= nch) return;
        unsigned char* st = sm + (n & 1) * Sm::STAGE;
        const float* rec = rec_of(n);
        uint64_t* bar = &bar_full[n & 1];
        mbar_arrive_expect_tx(bar, Sm::TX_BYTES);
        bulk_load(st + Sm::SP, rec + R::P, 16384, bar);
        bulk_load(st + Sm::SU0, rec + R::U0 + (size_t)(j0 / 32) * 2048, (NS / 32) * 8192, bar);
        bulk_load(st + Sm::SGC, rec + R::GC, DK * 4, bar);
    };
    // this thread's A-operand values of chunk n: its [W; Q~] row (DK/2 channels)
    // and, on channel lanes, its K^^T row (32 tokens)
    float wq[DK / 2], kh[32];
    auto load_a = [&](int n) {
        if (n >= nch) return;
        const float* rec = rec_of(n);
        const float* a = rec + R::WQ + (size_t)lane_row * DK + wg * (DK / 2);
#pragma unroll
        for (int j = 0; j < DK / 2; j += 4) {
            const float4 x = *reinterpret_cast<const float4*>(a + j);
            wq[j] = x.x; wq[j + 1] = x.y; wq[j + 2] = x.z; wq[j + 3] = x.w;
        }
        if (chan) {
            const float* b = rec + R::KHT + (size_t)lane_row * kChunk + 32 * wg;
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 x = *reinterpret_cast<const float4*>(b + j);
                kh[j] = x.x; kh[j + 1] = x.y; kh[j + 2] = x.z; kh[j + 3] = x.w;
            }
        }
    };
    auto put_wq = [&]() {   // -> TMEM (hi | lo), all lanes
#pragma unroll
        for (int j = 0; j < DK / 2; j += 32) {
            float hi[32], lo[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) split_tf32_(wq[j + e], hi[e], lo[e]);
            tmem_st32_sync(WQA + lane_base + wg * (DK / 2) + j, hi);
            tmem_st32_sync(WQA + DK + lane_base + wg * (DK / 2) + j, lo);
        }
    };
    auto put_kh = [&]() {   // -> TMEM (hi | lo), channel lanes (warp-uniform)
        if ((warp & 3) * 32 < DK) {
            float hi[32], lo[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) split_tf32_(kh[e], hi[e], lo[e]);
            tmem_st32_sync(KHA + lane_base + 32 * wg, hi);
            tmem_st32_sync(KHA + 64 + lane_base + 32 * wg, lo);
        }
    };
    // S^T (hi | lo) from this thread's CPT state columns (channel = lane_row)
    auto put_st = [&](const float* v) {
        const int c = lane_row;
#pragma unroll
        for (int e = 0; e < CPT; ++e) {
            float hi, lo;
            split_tf32_(v[e], hi, lo);
            const uint32_t off = (uint32_t)(c >> 5) * Sm::ST_TILE + sw128_offset(cb + e, (c & 31) * 4);
            *reinterpret_cast<float*>(sm + Sm::ST + off) = hi;
            *reinterpret_cast<float*>(sm + Sm::ST + Sm::ST_HALF + off) = lo;
        }
    };
    // CPT consecutive TMEM columns of this thread's lane, waited for
    auto ld_cols = [&](uint32_t taddr, float* v) {
#pragma unroll
        for (int c = 0; c < CPT; c += 16) {
            float t[16];
            tmem_ld16(taddr + c, t);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) v[c + i] = t[i];
        }
    };
    auto st_cols = [&](uint32_t taddr, const float* v) {
#pragma unroll
        for (int c = 0; c < CPT; c += 16) {
            float t[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) t[i] = v[c + i];
            tmem_st16(taddr + c, t);
        }
    };
    auto write_o = [&](int n) {   // output rows (lanes 64..127) of chunk n from its R3
        const int r = lane_row - 64;
        const int tok = tok_begin + n * kChunk + r;
        float v[CPT];
        ld_cols(r3(n) + lane_base + cb, v);
        if (tok < tok_end) {
            float* dst = o + ((size_t)tok * H + h) * DV + j0 + cb;
#pragma unroll
            for (int i = 0; i < CPT; i += 4)
                *reinterpret_cast<float4*>(dst + i) = make_float4(scale * v[i], scale * v[i + 1], scale * v[i + 2], scale * v[i + 3]);
        }
    };

    // initial state slice -> TMEM accumulator and S^T
    if (chan) {
        float v[CPT];
#pragma unroll
        for (int i = 0; i < CPT; i += 4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (initial_state)
                x = *reinterpret_cast<const float4*>(initial_state + state_off + (size_t)lane_row * DV + j0 + cb + i);
            v[i] = x.x; v[i + 1] = x.y; v[i + 2] = x.z; v[i + 3] = x.w;
        }
        st_cols(SACC + lane_base + cb, v);
        put_st(v);
    }
    if (tid == 0) {
        issue(0);
        issue(1);
    }
    load_a(0);
    if (nch > 0) put_wq();
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    bool aborted = false;
    uint32_t mma_phase = 0;
    int mma_pending = 0;
    int copies_issued = nch < 2 ? nch : 2, copies_done = 0;
    auto wait_mma = [&]() -> bool {
        const bool ok = mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        if (__syncthreads_or(!ok)) return false;
        mma_phase ^= 1;
        mma_pending = 0;
        tc_fence_after();
        return true;
    };
    for (int n = 0; n < nch; ++n) {
        const int b = n & 1;
        unsigned char* st = sm + b * Sm::STAGE;
        {
            const bool ok = mbar_wait_cycles(&bar_full[b], (n >> 1) & 1, kWaitCycles);
            if (__syncthreads_or(!ok)) { aborted = true; break; }
        }
        copies_done = n + 1;
        const uint32_t R3 = r3(n);
        // MMA3: [W; Q~] S -> R3 (split tf32; K = DK channels)
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc = instr_desc(kFmtTF32, 128, NS);
            const uint32_t sb = smem_u32(sm + Sm::ST);
#pragma unroll
            for (int pass = 0; pass < 3; ++pass) {
                const uint32_t acol = pass == 1 ? DK : 0;
                const uint32_t boff = pass == 0 ? Sm::ST_HALF : 0;
#pragma unroll
                for (int kk = 0; kk < DK / 8; ++kk)
                    mma_tf32_ts(R3, WQA + acol + kk * 8,
                                smem_desc(sb + boff + (kk >> 2) * Sm::ST_TILE + (kk & 3) * 32, 16, 1024, kLayoutSW128), idesc,
                                (pass | kk) != 0);
            }
            mma_commit(&bar_mma);
        }
        mma_pending = 1;
        // meanwhile: K^^T of this chunk -> TMEM (MMA5 of the previous chunk is
        // done), the next chunk's A operands into registers, P (hi | lo) into the
        // [*; P] tiles, S <- Diag(gamma_C) S, the previous chunk's output rows
        put_kh();
        load_a(n + 1);
        {
            const float* sp = reinterpret_cast<const float*>(st + Sm::SP);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int idx = tid + 256 * i;            // 16-byte chunk of the two P tiles
                const int th = idx >> 9, within = idx & 511;
                const float4 x = *reinterpret_cast<const float4*>(sp + idx * 4);
                float4 hi, lo;
                split_tf32_(x.x, hi.x, lo.x);
                split_tf32_(x.y, hi.y, lo.y);
                split_tf32_(x.z, hi.z, lo.z);
                split_tf32_(x.w, hi.w, lo.w);
                const uint32_t off = 8192u + (uint32_t)within * 16u;   // rows 64..127 of the tile
                *reinterpret_cast<float4*>(sm + Sm::PA + th * 16384 + off) = hi;
                *reinterpret_cast<float4*>(sm + Sm::PA + (2 + th) * 16384 + off) = lo;
            }
        }
        if (chan) {
            const float gc = reinterpret_cast<const float*>(st + Sm::SGC)[lane_row];
            float v[CPT];
            ld_cols(SACC + lane_base + cb, v);
#pragma unroll
            for (int i = 0; i < CPT; ++i) v[i] *= gc;
            st_cols(SACC + lane_base + cb, v);
        }
        if (NB == 2 && n > 0 && lane_row >= 64) write_o(n - 1);
        tmem_wait_st();
        if (!wait_mma()) { aborted = true; break; }

        // U = U0 - W S (lanes 0..63 = tokens) -> U^T (hi | lo)
        if (lane_row < 64) {
            const int r = lane_row;
            float v[CPT];
            ld_cols(R3 + lane_base + cb, v);
#pragma unroll
            for (int i4 = 0; i4 < CPT / 4; ++i4) {
                const int col = (int)cb + 4 * i4;             // column in the slice; 32-column record tiles
                const float4 u0 = *reinterpret_cast<const float4*>(st + Sm::SU0 + (col >> 5) * 8192 +
                                                                   sw128_offset(r, ((col & 31) >> 2) * 16));
                const float u[4] = {u0.x - v[4 * i4], u0.y - v[4 * i4 + 1], u0.z - v[4 * i4 + 2], u0.w - v[4 * i4 + 3]};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float hi, lo;
                    split_tf32_(u[e], hi, lo);
                    const uint32_t off = (uint32_t)(r >> 5) * 16384u + sw128_offset(col + e, (r & 31) * 4);
                    *reinterpret_cast<float*>(sm + Sm::PA + off) = hi;
                    *reinterpret_cast<float*>(sm + Sm::PA + Sm::UT_HALF + off) = lo;
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // MMA4: [*; P] U += R3 ; MMA5: K^^T U += S  (split tf32; K = 64 tokens)
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc = instr_desc(kFmtTF32, 128, NS);
            const uint32_t pa = smem_u32(sm + Sm::PA), ub = pa;
#pragma unroll
            for (int pass = 0; pass < 3; ++pass) {
                const uint32_t pofs = pass == 1 ? 2 * 16384 : 0;       // P lo on pass 1
                const uint32_t kcol = pass == 1 ? 64 : 0;              // K^^T lo on pass 1
                const uint32_t uofs = pass == 0 ? Sm::UT_HALF : 0;     // U lo on pass 0
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t bdesc = smem_desc(ub + uofs + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kLayoutSW128);
                    mma_tf32(R3, smem_desc(pa + pofs + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kLayoutSW128),
                             bdesc, idesc, true);
                    mma_tf32_ts(SACC, KHA + kcol + kk * 8, bdesc, idesc, true);
                }
            }
            mma_commit(&bar_mma);
        }
        mma_pending = 1;
        // meanwhile: the next chunk's [W; Q~] -> TMEM (MMA3 is done with it), and
        // this stage's records are consumed
        if (n + 1 < nch) put_wq();
        tmem_wait_st();
        if (tid == 0) {
            fence_proxy_async_smem();
            issue(n + 2);
        }
        if (n + 2 < nch) copies_issued = n + 3;
        if (!wait_mma()) { aborted = true; break; }
        // with one R3: this chunk's output rows before the next MMA3
        if (NB == 1 && lane_row >= 64) write_o(n);
        // next state -> S^T (the serial path)
        if (chan) {
            float v[CPT];
            ld_cols(SACC + lane_base + cb, v);
            put_st(v);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (aborted) {
        if (tid == 0) {
            flag_error(hdr, kStatusTimeout);
            if (mma_pending) (void)mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
            for (int j = copies_done; j < copies_issued; ++j)
                (void)mbar_wait_cycles(&bar_full[j & 1], (j >> 1) & 1, kWaitCycles / 8);
        }
    } else {
        if (NB == 2 && nch > 0 && lane_row >= 64) write_o(nch - 1);
        if (final_state && chan) {
            float v[CPT];
            ld_cols(SACC + lane_base + cb, v);
            float* dst = final_state + state_off + (size_t)lane_row * DV + j0 + cb;
#pragma unroll
            for (int i = 0; i < CPT; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int DK, int DV, int NS>
cudaError_t launch_inter_f32_tc_ns(const ChunkArgs& a) {
    ChunkMap map{a.cu_seqlens, a.chunk_offsets, a.num_seqs, a.T, a.fixed_chunks_per_seq};
    auto kern = inter_chunk_f32_tc_kernel<DK, DV, NS>;
    const int smem = (int)F32K2Smem<DK, DV, NS>::END + 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((size_t)a.num_seqs * a.H * (DV / NS));
    kern<<<grid, 256, smem, a.stream>>>(a.initial_state, a.final_state, static_cast<float*>(a.o), map,
                                        static_cast<WsHeader*>(a.ws_header), static_cast<const float*>(a.records),
                                        a.H, a.max_chunks, a.scale);
    return cudaGetLastError();
}

// 32-column slices while they all fit in one wave of CTAs (one per SM), else 64.
template <int DK, int DV>
cudaError_t launch_inter_f32_tc_t(const ChunkArgs& a) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long chains = (long long)a.num_seqs * a.H;
    if (chains * (DV / 32) <= sms) return launch_inter_f32_tc_ns<DK, DV, 32>(a);
    return launch_inter_f32_tc_ns<DK, DV, 64>(a);
}

}  // namespace

cudaError_t launch_chunk_inter_f32_tc(const ChunkArgs& a) {
    if (a.num_seqs == 0) return cudaSuccess;
    if (a.dk == 128 && a.dv == 128) return launch_inter_f32_tc_t<128, 128>(a);
    if (a.dk == 128 && a.dv == 64) return launch_inter_f32_tc_t<128, 64>(a);
    if (a.dk == 64 && a.dv == 128) return launch_inter_f32_tc_t<64, 128>(a);
    if (a.dk == 64 && a.dv == 64) return launch_inter_f32_tc_t<64, 64>(a);
    return cudaErrorInvalidValue;
}

}  // namespace kda
