// kda_chunk_tc.cu -- chunkwise KDA forward on the sm_100a tensor cores
// (tcgen05 + TMEM, TMA / bulk-copy fed) for bf16 inputs.
//
// The chunk algebra is the one of kda_chunk_simt.cu (unrolling the daiw.net
// update equation, section "KDA 的更新式", over chunks of 64 tokens; chunk-wise
// parallel form of the kongchang.com page, section "硬件效率的优化策略"):
//
//   A_{ri} = beta_r <k_r e^{g_r-g_m}, k_i e^{g_m-g_i}>  (i < r),  T = (I + A)^{-1}
//   P_{ri} =        <q_r e^{g_r-g_m}, k_i e^{g_m-g_i}>  (i <= r)
//   W  = T diag(beta) (k e^{g}),   U0 = T diag(beta) V,   Q~ = q e^{g},
//   K^ = k e^{g_{L-1} - g},        gC = e^{g_{L-1}}
//   U = U0 - W S,   O = dk^{-1/2} (Q~ S + P U),   S' = Diag(gC) S + K^^T U
//
// K1 intra_chunk_tc (one CTA per (chunk, head), all chunks in parallel):
//   TMA loads q, k, v (bf16, 128-byte swizzled) and log_alpha (fp32) of the
//   chunk; one thread per key channel forms the cumulative decay and the
//   decayed operands; a tf32 MMA gives [A; P] = [K~m; Q~m] K-m^T in TMEM; T is
//   formed by forward substitution (one column per thread); an fp16 MMA gives
//   [W | U0] = T diag(beta) [K~ | V].  The chunk's intermediates go to the
//   workspace in fp16, already laid out as the operand tiles K2's MMAs read.
// K2 inter_chunk_tc (one CTA per (sequence, head, 64-wide value slice),
//   serial over the sequence's chunks): the fp32 state slice lives in TMEM
//   for the whole sequence; each chunk's intermediates arrive by bulk copy into
//   a double buffer; per chunk three MMA groups: [W; Q~] S, then
//   [*; P] U and K^^T U accumulated onto the TMEM accumulators.
//
// Precision: tf32 operands (rounded to nearest) for A and P, whose factors can
// exceed the fp16 range; fp16 (10-bit mantissa, like tf32) for every other
// operand and intermediate, all accumulation in fp32.  fp16 values above 65000
// in magnitude set KDA_ERR_RANGE in the workspace status.
//
// All waits are bounded (about one second of SM clock); a CTA that gives up
// records KDA_ERR_TIMEOUT, waits (bounded) for its own outstanding MMAs and
// copies, frees its tensor memory and returns.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kda_common.cuh"
#include "kda_launch.h"
#include "ptx.cuh"

namespace kda {
namespace {

using namespace ptx;

constexpr long long kWaitCycles = 2000000000LL;  // ~1 s at 2 GHz
constexpr float kF16Limit = 65000.f;

// Byte offset of fp16 element (row, col) in a stack of 128-byte-swizzled
// tiles that hold 64 columns per tile; `tile_bytes` apart.
__device__ __forceinline__ uint32_t h_off(uint32_t row, uint32_t col, uint32_t tile_bytes) {
    return (col >> 6) * tile_bytes + sw128_offset(row, (col & 63u) * 2u);
}
// Same for fp32 elements (32 columns per 128-byte row).
__device__ __forceinline__ uint32_t f_off(uint32_t row, uint32_t col, uint32_t tile_bytes) {
    return (col >> 5) * tile_bytes + sw128_offset(row, (col & 31u) * 4u);
}

__device__ __forceinline__ void flag_error(WsHeader* hdr, int code) {
    atomicCAS(&hdr->runtime_err, 0, code);
}

// ---------------------------------------------------------- record ------
// Per (head, chunk), fp16 unless noted, every tile 128-byte swizzled:
//   WQ  K-major operand, 128 rows (0..63 W, 64..127 Q~), K = dk: dk/64 tiles of 16 KB
//   KH  K^ with rows = token, 64 channels per tile: dk/64 tiles of 8 KB (MN-major A of K^^T U)
//   P   K-major rows = token r, K = token i: one 8 KB tile
//   U0  rows = token, 64 value columns per tile: dv/64 tiles of 8 KB
//   GC  fp32 [dk]
template <int DK, int DV>
struct TcRec {
    static constexpr uint32_t WQ = 0, WQ_BYTES = (DK / 64) * 16384;
    static constexpr uint32_t KH = WQ + WQ_BYTES, KH_BYTES = (DK / 64) * 8192;
    static constexpr uint32_t P = KH + KH_BYTES, P_BYTES = 8192;
    static constexpr uint32_t U0 = P + P_BYTES, U0_BYTES = (DV / 64) * 8192;
    static constexpr uint32_t GC = U0 + U0_BYTES, GC_BYTES = DK * 4;
    static constexpr uint32_t BYTES = (GC + GC_BYTES + 1023) / 1024 * 1024;
};

// ---------------------------------------------------------------- K1 ----
template <int DK, int DV>
struct K1Smem {
    static constexpr uint32_t KS = 0;                           // k tiles (bf16 -> fp16 K~ in place)
    static constexpr uint32_t VS = KS + (DK / 64) * 8192;       // v tiles (bf16 -> fp16 in place)
    static constexpr uint32_t QS = VS + (DV / 64) * 8192;       // q tiles (bf16)
    static constexpr uint32_t LAS = QS + (DK / 64) * 8192;      // log_alpha [64][DK] fp32, dense
    static constexpr uint32_t OPA = LAS + 64 * DK * 4;          // tf32 [K~m; Q~m]: DK/32 tiles of 16 KB
    static constexpr uint32_t OPB = OPA + (DK / 32) * 16384;    // tf32 K-m: DK/32 tiles of 8 KB
    static constexpr uint32_t END = OPB + (DK / 32) * 8192;
    static constexpr uint32_t AM = QS;   // after the decay pass: A in fp32 [64][65]
    static constexpr uint32_t TP = OPB;  // after MMA1: T diag(beta) fp16, K-major 128 x 64 tokens
    static constexpr uint32_t TX_BYTES = (2 * (DK / 64) + DV / 64) * 8192 + 64 * DK * 4;
    static_assert(QS + 64 * 65 * 4 <= OPA, "A matrix alias");
    static_assert(TP + 16384 <= END, "T alias");
};

template <int DK, int DV>
__global__ void __launch_bounds__(256, 1)
intra_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_la,
                      const float* __restrict__ beta, ChunkMap map, WsHeader* hdr,
                      unsigned char* __restrict__ records, int H, size_t max_chunks)
{
    using Sm = K1Smem<DK, DV>;
    using R = TcRec<DK, DV>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar_load, bar_mma;
    __shared__ uint32_t s_tmem;
    __shared__ float s_beta[kChunk];

    if (hdr->status != kStatusOk) return;
    const int c = blockIdx.x, h = blockIdx.y;
    if (c >= hdr->num_chunks) return;
    int seq, tok0, L;
    map.locate(c, seq, tok0, L);
    const int tid = threadIdx.x, warp = tid >> 5;
    unsigned char* rec = records + ((size_t)h * max_chunks + c) * R::BYTES;

    if (tid == 0) {
        mbar_init(&bar_load, 1);
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
    const uint32_t R1 = tmem;         // [A; P]      128 lanes x 64 columns (fp32)
    const uint32_t R2 = tmem + 128;   // [W | U0]    128 lanes x (DK + DV) columns
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;

    if (tid == 0) {
        mbar_arrive_expect_tx(&bar_load, Sm::TX_BYTES);
#pragma unroll
        for (int b = 0; b < DK / 64; ++b) tma_load_3d(sm + Sm::KS + b * 8192, &tm_k, &bar_load, b * 64, h, tok0);
#pragma unroll
        for (int b = 0; b < DV / 64; ++b) tma_load_3d(sm + Sm::VS + b * 8192, &tm_v, &bar_load, b * 64, h, tok0);
#pragma unroll
        for (int b = 0; b < DK / 64; ++b) tma_load_3d(sm + Sm::QS + b * 8192, &tm_q, &bar_load, b * 64, h, tok0);
        tma_load_3d(sm + Sm::LAS, &tm_la, &bar_load, 0, h, tok0);
    }
    if (tid >= 192) {
        const int r = tid - 192;
        s_beta[r] = (r < L) ? beta[(size_t)(tok0 + r) * H + h] : 0.f;
    }
    bool ok = mbar_wait_cycles(&bar_load, 0, kWaitCycles);
    bool aborted = __syncthreads_or(!ok);
    int mma_issued = 0;   // commits issued on bar_mma (uniform across the CTA)
    float range_max = 0.f;

    if (!aborted) {
        // ---- decay pass: one thread per key channel ------------------------
        if (tid < DK) {
            const int ch = tid;
            const float* las = reinterpret_cast<const float*>(sm + Sm::LAS);
            float g[kChunk];
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < kChunk; ++r) {
                acc += (r < L) ? las[r * DK + ch] : 0.f;
                g[r] = acc;
            }
            float gm = g[0], gl = g[0];
#pragma unroll
            for (int r = 0; r < kChunk; ++r) {
                if (r == ((L - 1) >> 1)) gm = g[r];
                if (r == L - 1) gl = g[r];
            }
            const float egm = __expf(gm), eglm = __expf(gl - gm);
#pragma unroll
            for (int r = 0; r < kChunk; ++r) {
                const uint32_t ho = h_off(r, ch, 8192);
                float kk = 0.f, qq = 0.f;
                if (r < L) {
                    kk = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + Sm::KS + ho));
                    qq = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + Sm::QS + ho));
                }
                const float em = __expf(g[r] - gm);   // e^{g_r - g_m}
                const float eb = __expf(gm - g[r]);   // e^{g_m - g_r}
                const float e0 = egm * em;            // e^{g_r}
                const float eh = eglm * eb;           // e^{g_{L-1} - g_r}
                *reinterpret_cast<float*>(sm + Sm::OPA + f_off(r, ch, 16384)) = round_tf32(kk * em);
                *reinterpret_cast<float*>(sm + Sm::OPA + f_off(64 + r, ch, 16384)) = round_tf32(qq * em);
                *reinterpret_cast<float*>(sm + Sm::OPB + f_off(r, ch, 8192)) = round_tf32(kk * eb);
                *reinterpret_cast<__half*>(sm + Sm::KS + ho) = __float2half_rn(kk * e0);
                const float qt = qq * e0, kh = kk * eh;
                *reinterpret_cast<__half*>(rec + R::WQ + h_off(64 + r, ch, 16384)) = __float2half_rn(qt);
                *reinterpret_cast<__half*>(rec + R::KH + ho) = __float2half_rn(kh);
            }
            reinterpret_cast<float*>(rec + R::GC)[ch] = expf(gl);
        } else {
            // v: bf16 -> fp16 in place (same swizzled slot), zero beyond the chunk
            for (int idx = tid - DK; idx < kChunk * DV; idx += 256 - DK) {
                const int r = idx / DV, j = idx - r * DV;
                const uint32_t o = Sm::VS + h_off(r, j, 8192);
                const float x = (r < L) ? __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + o)) : 0.f;
                range_max = fmaxf(range_max, fabsf(x));
                *reinterpret_cast<__half*>(sm + o) = __float2half_rn(x);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- MMA1 (tf32): [K~m; Q~m] K-m^T -> R1 ---------------------------
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc = instr_desc(kFmtTF32, 128, 64);
            const uint32_t a0 = smem_u32(sm + Sm::OPA), b0 = smem_u32(sm + Sm::OPB);
#pragma unroll
            for (int kb = 0; kb < DK / 32; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_tf32(R1, smem_desc(a0 + kb * 16384 + ks * 32, 16, 1024, kLayoutSW128),
                             smem_desc(b0 + kb * 8192 + ks * 32, 16, 1024, kLayoutSW128), idesc,
                             (kb | ks) != 0);
            mma_commit(&bar_mma);
        }
        mma_issued = 1;
        ok = mbar_wait_cycles(&bar_mma, 0, kWaitCycles);
        aborted = __syncthreads_or(!ok);
    }
    if (!aborted) {
        tc_fence_after();
        // ---- A to shared memory (rows 0..63), P to the record (rows 64..127)
        float* am = reinterpret_cast<float*>(sm + Sm::AM);  // [64][65]
        if (tid < 128) {
            float v[32];
            const int row = tid;   // TMEM lane = MMA row
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tmem_ld32_sync(R1 + lane_base + 32 * half, v);
                if (row < 64) {
                    const float b = s_beta[row];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int col = 32 * half + i;
                        am[row * 65 + col] = (col < row) ? b * v[i] : 0.f;
                    }
                } else {
                    const int r = row - 64;
#pragma unroll
                    for (int i8 = 0; i8 < 4; ++i8) {
                        __align__(16) __half hv[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int col = 32 * half + 8 * i8 + e;
                            hv[e] = __float2half_rn(col <= r ? v[8 * i8 + e] : 0.f);
                        }
                        *reinterpret_cast<uint4*>(rec + R::P + sw128_offset(r, (32 * half + 8 * i8) * 2)) =
                            *reinterpret_cast<const uint4*>(hv);
                    }
                }
            }
        }
        __syncthreads();

        // ---- T = (I + A)^{-1}: column tid by forward substitution ----------
        if (tid < kChunk) {
            float x[kChunk];
#pragma unroll
            for (int r = 0; r < kChunk; ++r) {
                float a0 = (r == tid) ? 1.f : 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                for (int i = 0; i + 3 < r; i += 4) {
                    a0 -= am[r * 65 + i] * x[i];
                    a1 -= am[r * 65 + i + 1] * x[i + 1];
                    a2 -= am[r * 65 + i + 2] * x[i + 2];
                    a3 -= am[r * 65 + i + 3] * x[i + 3];
                }
#pragma unroll
                for (int i = r & ~3; i < r; ++i) a0 -= am[r * 65 + i] * x[i];
                x[r] = (a0 + a1) + (a2 + a3);
            }
            const float bt = s_beta[tid];
#pragma unroll
            for (int r = 0; r < kChunk; ++r)   // T diag(beta), K-major row r, column tid
                *reinterpret_cast<__half*>(sm + Sm::TP + sw128_offset(r, tid * 2)) = __float2half_rn(x[r] * bt);
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- MMA2 (fp16): [T diag(beta); *] [K~ | V] -> R2 -----------------
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc = instr_desc(kFmtF16, 128, DK + DV, false, true);
            const uint32_t a0 = smem_u32(sm + Sm::TP), b0 = smem_u32(sm + Sm::KS);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_f16(R2, smem_desc(a0 + ks * 32, 16, 1024, kLayoutSW128),
                        smem_desc(b0 + ks * 2048, 8192, 1024, kLayoutSW128), idesc, ks != 0);
            mma_commit(&bar_mma);
        }
        mma_issued = 2;
        ok = mbar_wait_cycles(&bar_mma, 1, kWaitCycles);
        aborted = __syncthreads_or(!ok);
    }
    if (!aborted) {
        tc_fence_after();
        // ---- W and U0 (rows 0..63) to the record ---------------------------
        if (tid < 64) {
            const int r = tid;
#pragma unroll
            for (int cb = 0; cb < (DK + DV) / 32; ++cb) {
                float v[32];
                tmem_ld32_sync(R2 + lane_base + 32 * cb, v);
#pragma unroll
                for (int i8 = 0; i8 < 4; ++i8) {
                    __align__(16) __half hv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        range_max = fmaxf(range_max, fabsf(v[8 * i8 + e]));
                        hv[e] = __float2half_rn(v[8 * i8 + e]);
                    }
                    const int col = 32 * cb + 8 * i8;
                    unsigned char* dst = (col < DK) ? rec + R::WQ + h_off(r, col, 16384)
                                                    : rec + R::U0 + h_off(r, col - DK, 8192);
                    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(hv);
                }
            }
        }
    } else {
        if (tid == 0) flag_error(hdr, kStatusTimeout);
        // let this CTA's own copies and MMAs finish (bounded) before freeing
        (void)mbar_wait_cycles(&bar_load, 0, kWaitCycles);
        if (mma_issued > 0) (void)mbar_wait_cycles(&bar_mma, (uint32_t)(mma_issued - 1), kWaitCycles);
    }
    if (range_max > kF16Limit) flag_error(hdr, kStatusRange);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- K2 ----
constexpr int kSliceTc = 64;   // value columns per inter-chunk CTA

template <int DK, int DV>
struct K2Smem {
    using R = TcRec<DK, DV>;
    // one stage: [WQ][KH][P][U0 slice][GC]; P directly after KH, so the
    // 128-row A operand [*; P] reads the tail of KH as its (unused) rows 0..63
    static constexpr uint32_t WQ = 0;
    static constexpr uint32_t KH = WQ + R::WQ_BYTES;
    static constexpr uint32_t P = KH + R::KH_BYTES;
    static constexpr uint32_t U0 = P + 8192;
    static constexpr uint32_t GC = U0 + 8192;
    static constexpr uint32_t STAGE = (GC + DK * 4 + 1023) / 1024 * 1024;
    static constexpr uint32_t S16 = 2 * STAGE;              // fp16 state slice, rows = key channel
    static constexpr uint32_t U16 = S16 + 128 * 128;        // fp16 U, rows = token
    static constexpr uint32_t END = U16 + 8192;
    static constexpr uint32_t TX_BYTES = R::WQ_BYTES + R::KH_BYTES + 8192 + 8192 + DK * 4;
};

template <int DK, int DV>
__global__ void __launch_bounds__(128, 1)
inter_chunk_tc_kernel(const float* __restrict__ initial_state, float* __restrict__ final_state,
                      __nv_bfloat16* __restrict__ o, ChunkMap map, WsHeader* hdr,
                      const unsigned char* __restrict__ records, int H, size_t max_chunks, float scale)
{
    using Sm = K2Smem<DK, DV>;
    using R = TcRec<DK, DV>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar_full[2], bar_mma;
    __shared__ uint32_t s_tmem;

    if (hdr->status != kStatusOk) return;
    const int s = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * kSliceTc;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int first = map.seq_first_chunk(s), nch = map.seq_num_chunks(s);
    const int tok_begin = map.seq_token_begin(s), tok_end = map.seq_token_end(s);
    const size_t state_off = ((size_t)s * H + h) * DK * DV;

    if (tid == 0) {
        mbar_init(&bar_full[0], 1);
        mbar_init(&bar_full[1], 1);
        mbar_init(&bar_mma, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&s_tmem, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const uint32_t R3 = tmem;        // [W S; Q~ S + P U]   128 lanes x 64
    const uint32_t SACC = tmem + 64; // state slice (fp32)  lanes = key channel
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    float range_max = 0.f;

    auto issue = [&](int n) {   // bulk-copy chunk n's intermediates into stage n & 1
        if (n >= nch) return;
        unsigned char* st = sm + (n & 1) * Sm::STAGE;
        const unsigned char* rec = records + ((size_t)h * max_chunks + first + n) * R::BYTES;
        uint64_t* bar = &bar_full[n & 1];
        mbar_arrive_expect_tx(bar, Sm::TX_BYTES);
        bulk_load(st + Sm::WQ, rec + R::WQ, R::WQ_BYTES, bar);
        bulk_load(st + Sm::KH, rec + R::KH, R::KH_BYTES, bar);
        bulk_load(st + Sm::P, rec + R::P, 8192, bar);
        bulk_load(st + Sm::U0, rec + R::U0 + (j0 / 64) * 8192, 8192, bar);
        bulk_load(st + Sm::GC, rec + R::GC, DK * 4, bar);
    };

    // initial state slice -> TMEM accumulator and fp16 operand copy
    if (tid < DK) {
        float v[32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (initial_state)
                    x = *reinterpret_cast<const float4*>(initial_state + state_off + (size_t)tid * DV + j0 + 32 * half + i);
                v[i] = x.x; v[i + 1] = x.y; v[i + 2] = x.z; v[i + 3] = x.w;
            }
            tmem_st32_sync(SACC + lane_base + 32 * half, v);
#pragma unroll
            for (int i8 = 0; i8 < 4; ++i8) {
                __align__(16) __half hv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    range_max = fmaxf(range_max, fabsf(v[8 * i8 + e]));
                    hv[e] = __float2half_rn(v[8 * i8 + e]);
                }
                *reinterpret_cast<uint4*>(sm + Sm::S16 + sw128_offset(tid, (32 * half + 8 * i8) * 2)) =
                    *reinterpret_cast<const uint4*>(hv);
            }
        }
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
    for (int n = 0; n < nch && !aborted; ++n) {
        const int b = n & 1;
        unsigned char* st = sm + b * Sm::STAGE;
        bool ok = mbar_wait_cycles(&bar_full[b], (n >> 1) & 1, kWaitCycles);
        if (__syncthreads_or(!ok)) { aborted = true; break; }

        // MMA3: [W; Q~] S -> R3
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc = instr_desc(kFmtF16, 128, kSliceTc, false, true);
            const uint32_t a0 = smem_u32(st + Sm::WQ), b0 = smem_u32(sm + Sm::S16);
#pragma unroll
            for (int kb = 0; kb < DK / 64; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(R3, smem_desc(a0 + kb * 16384 + ks * 32, 16, 1024, kLayoutSW128),
                            smem_desc(b0 + kb * 8192 + ks * 2048, 8192, 1024, kLayoutSW128), idesc,
                            (kb | ks) != 0);
            mma_commit(&bar_mma);
        }
        // meanwhile: S_acc <- Diag(gC) S_acc (MMA3 reads the fp16 copy, not S_acc)
        if (tid < DK) {
            const float gc = reinterpret_cast<const float*>(st + Sm::GC)[tid];
            float v[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tmem_ld32_sync(SACC + lane_base + 32 * half, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= gc;
                tmem_st32_sync(SACC + lane_base + 32 * half, v);
            }
        }
        ok = mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        mma_phase ^= 1;
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        tc_fence_after();

        // U = U0 - W S  (rows 0..63 = tokens), fp16 -> U16
        if (tid < 64) {
            const int r = tid;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
                tmem_ld32_sync(R3 + lane_base + 32 * half, v);
#pragma unroll
                for (int i8 = 0; i8 < 4; ++i8) {
                    const uint32_t off = sw128_offset(r, (32 * half + 8 * i8) * 2);
                    const uint4 u0raw = *reinterpret_cast<const uint4*>(st + Sm::U0 + off);
                    const __half* u0 = reinterpret_cast<const __half*>(&u0raw);
                    __align__(16) __half hv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float u = __half2float(u0[e]) - v[8 * i8 + e];
                        range_max = fmaxf(range_max, fabsf(u));
                        hv[e] = __float2half_rn(u);
                    }
                    *reinterpret_cast<uint4*>(sm + Sm::U16 + off) = *reinterpret_cast<const uint4*>(hv);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // MMA4: [*; P] U += R3 ; MMA5: K^^T U += S_acc
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc = instr_desc(kFmtF16, 128, kSliceTc, false, true);
            constexpr uint32_t idesc_t = instr_desc(kFmtF16, 128, kSliceTc, true, true);
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
        ok = mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        mma_phase ^= 1;
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        tc_fence_after();
        if (tid == 0) {
            fence_proxy_async_smem();
            issue(n + 2);   // this stage is no longer read
        }

        // O = scale (Q~ S + P U): rows 64..127
        if (tid >= 64) {
            const int r = tid - 64;
            const int tok = tok_begin + n * kChunk + r;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
                tmem_ld32_sync(R3 + lane_base + 32 * half, v);
                if (tok < tok_end) {
                    __nv_bfloat16* dst = o + ((size_t)tok * H + h) * DV + j0 + 32 * half;
#pragma unroll
                    for (int i8 = 0; i8 < 4; ++i8) {
                        __align__(16) __nv_bfloat16 bv[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) bv[e] = __float2bfloat16_rn(scale * v[8 * i8 + e]);
                        *reinterpret_cast<uint4*>(dst + 8 * i8) = *reinterpret_cast<const uint4*>(bv);
                    }
                }
            }
        }
        // next state's fp16 operand copy
        if (tid < DK) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
                tmem_ld32_sync(SACC + lane_base + 32 * half, v);
#pragma unroll
                for (int i8 = 0; i8 < 4; ++i8) {
                    __align__(16) __half hv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        range_max = fmaxf(range_max, fabsf(v[8 * i8 + e]));
                        hv[e] = __float2half_rn(v[8 * i8 + e]);
                    }
                    *reinterpret_cast<uint4*>(sm + Sm::S16 + sw128_offset(tid, (32 * half + 8 * i8) * 2)) =
                        *reinterpret_cast<const uint4*>(hv);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (aborted) {
        if (tid == 0) flag_error(hdr, kStatusTimeout);
        // let MMAs and copies this CTA issued finish before its memory goes away
        (void)mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        for (int b = 0; b < 2; ++b) (void)mbar_wait_cycles(&bar_full[b], 0, kWaitCycles / 8);
    } else if (final_state && tid < DK) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float v[32];
            tmem_ld32_sync(SACC + lane_base + 32 * half, v);
            float* dst = final_state + state_off + (size_t)tid * DV + j0 + 32 * half;
#pragma unroll
            for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
    }
    if (range_max > kF16Limit) flag_error(hdr, kStatusRange);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

// ------------------------------------------------------------- host -----
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// [ntok, H, d] row-major tensor; boxes of `box_inner` x 1 head x 64 tokens.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, int d, int H,
              int ntok, int box_inner, CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)ntok};
    cuuint64_t strides[2] = {(cuuint64_t)d * elem_bytes, (cuuint64_t)H * d * elem_bytes};
    cuuint32_t box[3] = {(cuuint32_t)box_inner, 1u, (cuuint32_t)kChunk};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK, int DV>
cudaError_t launch_intra_tc_t(const ChunkArgs& a) {
    if (a.max_chunks == 0) return cudaSuccess;
    const int ntok = a.cu_seqlens ? a.T : a.B * a.T;
    CUtensorMap mk, mv, mq, mla;
    if (!make_map(&mk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, a.H, ntok, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DV, a.H, ntok, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, a.H, ntok, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mla, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, DK, a.H, ntok, DK, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    ChunkMap map{a.cu_seqlens, a.chunk_offsets, a.num_seqs, a.T, a.fixed_chunks_per_seq};
    auto kern = intra_chunk_tc_kernel<DK, DV>;
    const int smem = (int)K1Smem<DK, DV>::END + 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)a.max_chunks, (unsigned)a.H);
    kern<<<grid, 256, smem, a.stream>>>(mk, mv, mq, mla, a.beta, map, static_cast<WsHeader*>(a.ws_header),
                                        static_cast<unsigned char*>(a.records), a.H, a.max_chunks);
    return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_inter_tc_t(const ChunkArgs& a) {
    ChunkMap map{a.cu_seqlens, a.chunk_offsets, a.num_seqs, a.T, a.fixed_chunks_per_seq};
    auto kern = inter_chunk_tc_kernel<DK, DV>;
    const int smem = (int)K2Smem<DK, DV>::END + 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)a.num_seqs, (unsigned)a.H, (unsigned)(DV / kSliceTc));
    kern<<<grid, 128, smem, a.stream>>>(a.initial_state, a.final_state, static_cast<__nv_bfloat16*>(a.o), map,
                                        static_cast<WsHeader*>(a.ws_header),
                                        static_cast<const unsigned char*>(a.records), a.H, a.max_chunks, a.scale);
    return cudaGetLastError();
}

#define KDA_TC_DISPATCH(FN, a)                                                  \
    do {                                                                       \
        if ((a).dk == 128 && (a).dv == 128) return FN<128, 128>(a);            \
        if ((a).dk == 128 && (a).dv == 64) return FN<128, 64>(a);              \
        if ((a).dk == 64 && (a).dv == 128) return FN<64, 128>(a);              \
        if ((a).dk == 64 && (a).dv == 64) return FN<64, 64>(a);                \
        return cudaErrorInvalidValue;                                          \
    } while (0)

}  // namespace

size_t tc_record_bytes(int dk, int dv) {
    if (dk == 128 && dv == 128) return TcRec<128, 128>::BYTES;
    if (dk == 128 && dv == 64) return TcRec<128, 64>::BYTES;
    if (dk == 64 && dv == 128) return TcRec<64, 128>::BYTES;
    if (dk == 64 && dv == 64) return TcRec<64, 64>::BYTES;
    return 0;
}

cudaError_t launch_chunk_intra_tc(const ChunkArgs& a) { KDA_TC_DISPATCH(launch_intra_tc_t, a); }

cudaError_t launch_chunk_inter_tc(const ChunkArgs& a) {
    if (a.num_seqs == 0) return cudaSuccess;
    KDA_TC_DISPATCH(launch_inter_tc_t, a);
}

}  // namespace kda
