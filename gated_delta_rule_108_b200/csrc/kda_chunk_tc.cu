// kda_chunk_tc.cu -- the backward of the chunkwise KDA forward on the sm_100a
// tensor cores (tcgen05 + TMEM, TMA / bulk-copy fed) for bf16 inputs, and the
// host side of the bf16 chunk kernels.
//
// The forward's chunk algebra (unrolling the daiw.net update equation, section
// "KDA 的更新式", over chunks of 64 tokens; chunk-wise parallel form of the
// kongchang.com page, section "硬件效率的优化策略"):
//
//   A_{ri} = beta_r <k_r e^{g_r-g_m}, k_i e^{g_m-g_i}>  (i < r),  T = (I + A)^{-1}
//   P_{ri} =        <q_r e^{g_r-g_m}, k_i e^{g_m-g_i}>  (i <= r)
//   W  = T diag(beta) (k e^{g}),   U0 = T diag(beta) V,   Q~ = q e^{g},
//   K^ = k e^{g_{L-1} - g},        gC = e^{g_{L-1}}
//   U = U0 - W S,   O = dk^{-1/2} (Q~ S + P U),   S' = Diag(gC) S + K^^T U
//
// The forward kernels are in kda_intra_tc.cu and kda_inter_tc.cu; in backward
// mode they also write what the kernels here read: fp16 tiles of T, K~ and V,
// the fp32 M = K_l K_r^T and a strong-decay flag per (head, chunk) (BwdTiles),
// and the fp32 state entering each chunk.  Here: the reversed chunk chain
// (KB3), then per (chunk, head) the products over the value dimension, the
// products through T, W and U0, and the split-factor products with the
// per-channel gradients (see each section).
//
// Precision: fp16 operands (10-bit mantissa) where the values stay in its range,
// tf32 where a factor e^{+-(g - g_m)} can leave it; fp32 accumulation.
//
// All waits are bounded (about one second of SM clock); a CTA that gives up
// records KDA_ERR_TIMEOUT, waits (bounded) for its own outstanding MMAs and
// copies, frees its tensor memory and returns.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>
#include <type_traits>

#include "kda_common.cuh"
#include "kda_launch.h"
#include "kda_tc_common.cuh"
#include "ptx.cuh"

namespace kda {
namespace {

using namespace ptx;

// ------------------------------------------- record stage (reversed chain) ----
constexpr int kSliceTc = 64;   // value columns per reversed-chain CTA

template <int DK, int DV>
struct K2Smem {
    using R = TcRec<DK, DV>;
    // one stage of a chunk's record: [WQ][KH][P][U0 slice][GC]; P directly after
    // KH, so a 128-row A operand [*; P] reads the tail of KH as its (unused) rows 0..63
    static constexpr uint32_t WQ = 0;
    static constexpr uint32_t KH = WQ + R::WQ_BYTES;
    static constexpr uint32_t P = KH + R::KH_BYTES;
    static constexpr uint32_t U0 = P + 8192;
    static constexpr uint32_t GC = U0 + 8192;
    static constexpr uint32_t STAGE = (GC + DK * 4 + 1023) / 1024 * 1024;
};

// --------------------------------------------------- backward KB3 (bf16) ----
// The backward's reversed chunk chain on the tensor cores (bf16 inputs), one
// CTA (8 warps) per (sequence, head, 64-wide value slice).  With D = c dO and
// dS' the cotangent of the state leaving chunk n:
//     dU = K^ dS' + P^T D        dS = Diag(gamma) dS' + Q~^T D + W^T (-dU)
// dS lives in TMEM (fp32) for the whole sequence with an fp16 copy in smem as
// the MMA operand, as the forward's state does; the records are the forward
// intra-chunk kernel's fp16 tiles and D is TMA-loaded from d_o (bf16) and
// converted in place.  dU and dS' of every chunk go out in fp32 for the
// per-chunk gradient kernel.
template <int DK, int DV>
struct B3Smem {
    using K2 = K2Smem<DK, DV>;                                  // record layout of a stage
    static constexpr uint32_t D = K2::STAGE;                    // cotangent tile: 64 tokens x 64 columns
    static constexpr uint32_t STAGE = K2::STAGE + 8192;
    static constexpr uint32_t DS16 = 2 * STAGE;                 // fp16 dS', rows = key channel
    static constexpr uint32_t DU16 = DS16 + 128 * 128;          // fp16 -dU, rows = token
    static constexpr uint32_t END = DU16 + 8192;
    static constexpr uint32_t TX_BYTES = TcRec<DK, DV>::WQ_BYTES + TcRec<DK, DV>::KH_BYTES + 8192 + DK * 4 + 8192;
};

template <int DK, int DV>
__global__ void __launch_bounds__(256, 1)
bwd_inter_tc_kernel(const __grid_constant__ CUtensorMap tm_do, const float* __restrict__ d_final_state,
                    float* __restrict__ d_initial_state, float* __restrict__ dS_end, float* __restrict__ dU_all,
                    ChunkMap map, WsHeader* hdr, const unsigned char* __restrict__ records, int H,
                    size_t max_chunks, float scale)
{
    using Sm = B3Smem<DK, DV>;
    using K2 = K2Smem<DK, DV>;
    using R = TcRec<DK, DV>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar_full[2], bar_mma;
    __shared__ uint32_t s_tmem;

    if (hdr->status != kStatusOk) return;
    const int s = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * kSliceTc;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int lane_row = (warp & 3) * 32 + (tid & 31);   // TMEM lane = MMA row
    const int wg = warp >> 2;                            // warpgroup: columns [32 wg, 32 wg + 32)
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
    const uint32_t RDU = tmem;          // [dU; *] 128 lanes x 64 columns
    const uint32_t SACC = tmem + 64;    // dS slice: lane = key channel
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    float range_max = 0.f;

    auto issue = [&](int n) {   // chunk n's records and cotangent tile into stage n & 1
        if (n < 0) return;
        unsigned char* st = sm + (n & 1) * Sm::STAGE;
        const unsigned char* rec = records + ((size_t)h * max_chunks + first + n) * R::BYTES;
        uint64_t* bar = &bar_full[n & 1];
        mbar_arrive_expect_tx(bar, Sm::TX_BYTES);
        bulk_load(st + K2::WQ, rec + R::WQ, R::WQ_BYTES, bar);
        bulk_load(st + K2::KH, rec + R::KH, R::KH_BYTES, bar);
        bulk_load(st + K2::P, rec + R::P, 8192, bar);
        bulk_load(st + K2::GC, rec + R::GC, DK * 4, bar);
        tma_load_3d(st + Sm::D, &tm_do, bar, j0, h, tok_begin + n * kChunk);
    };
    // fp16 copy of 32 columns of this thread's key channel of dS (row of DS16)
    auto put_ds16 = [&](const float (&v)[32]) {
#pragma unroll
        for (int i8 = 0; i8 < 4; ++i8) {
            __align__(16) __half2 hv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a = v[8 * i8 + 2 * e], b = v[8 * i8 + 2 * e + 1];
                range_max = fmaxf(range_max, fmaxf(fabsf(a), fabsf(b)));
                hv[e] = __floats2half2_rn(a, b);
            }
            *reinterpret_cast<uint4*>(sm + Sm::DS16 + sw128_offset(lane_row, (32 * wg + 8 * i8) * 2)) =
                *reinterpret_cast<const uint4*>(hv);
        }
    };

    // cotangent of the final state -> TMEM and its fp16 copy
    if (lane_row < DK) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (d_final_state)
                x = *reinterpret_cast<const float4*>(d_final_state + state_off + (size_t)lane_row * DV + j0 + 32 * wg + i);
            v[i] = x.x; v[i + 1] = x.y; v[i + 2] = x.z; v[i + 3] = x.w;
        }
        tmem_st32_sync(SACC + lane_base + 32 * wg, v);
        put_ds16(v);
    }
    if (tid == 0) {
        issue(nch - 1);
        issue(nch - 2);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    bool aborted = false;
    uint32_t mma_phase = 0;
    int mma_pending = 0;
    // the m-th chunk processed (n = nch - 1 - m) lands on bar_full[n & 1] with
    // phase parity (m >> 1) & 1; processed indices copies_done .. copies_issued - 1
    // are in flight (drained on abort)
    int copies_issued = nch < 2 ? nch : 2, copies_done = 0;
    for (int n = nch - 1; n >= 0; --n) {
        const int b = n & 1, m = nch - 1 - n;   // m-th chunk processed; stage b's (m >> 1)-th use
        unsigned char* st = sm + b * Sm::STAGE;
        const size_t item = (size_t)h * max_chunks + first + n;
        const int tok0 = tok_begin + n * kChunk;
        bool ok = mbar_wait_cycles(&bar_full[b], (m >> 1) & 1, kWaitCycles);
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        copies_done = m + 1;

        // D = c dO: bf16 -> fp16 in place; rows past the sequence are zero
        for (int it = tid; it < kChunk * 8; it += 256) {
            const int r = it >> 3, j8 = (it & 7) * 8;
            const uint32_t o = Sm::D + sw128_offset(r, j8 * 2);
            uint4 raw = *reinterpret_cast<const uint4*>(st + o);
            if (tok0 + r >= tok_end) raw = make_uint4(0, 0, 0, 0);
            const __nv_bfloat162* db = reinterpret_cast<const __nv_bfloat162*>(&raw);
            __align__(16) __half2 dh[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 x = __bfloat1622float2(db[e]);
                const float a = scale * x.x, c2 = scale * x.y;
                range_max = fmaxf(range_max, fmaxf(fabsf(a), fabsf(c2)));
                dh[e] = __floats2half2_rn(a, c2);
            }
            *reinterpret_cast<uint4*>(st + o) = *reinterpret_cast<const uint4*>(dh);
        }
        // dS' of this chunk out in fp32; then S_acc <- Diag(gamma) dS' (MMA-a reads the fp16 copy)
        if (lane_row < DK) {
            const float gc = reinterpret_cast<const float*>(st + K2::GC)[lane_row];
            float v[32];
            tmem_ld32_sync(SACC + lane_base + 32 * wg, v);
            float* dst = dS_end + (item * DK + lane_row) * DV + j0 + 32 * wg;
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                v[i] *= gc; v[i + 1] *= gc; v[i + 2] *= gc; v[i + 3] *= gc;
            }
            tmem_st32_sync(SACC + lane_base + 32 * wg, v);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // MMA-a: [K^; *] dS' + [P^T; *] D -> RDU
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc_k = instr_desc(kFmtF16, 128, kSliceTc, false, true);   // A K-major
            constexpr uint32_t idesc_m = instr_desc(kFmtF16, 128, kSliceTc, true, true);    // A MN-major
            const uint32_t kh = smem_u32(st + K2::KH), ds = smem_u32(sm + Sm::DS16);
            const uint32_t pa = smem_u32(st + K2::P), da = smem_u32(st + Sm::D);
#pragma unroll
            for (int kb = 0; kb < DK / 64; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(RDU, smem_desc(kh + kb * 8192 + ks * 32, 16, 1024, kLayoutSW128),
                            smem_desc(ds + kb * 8192 + ks * 2048, 8192, 1024, kLayoutSW128), idesc_k,
                            (kb | ks) != 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_f16(RDU, smem_desc(pa + ks * 2048, 8192, 1024, kLayoutSW128),
                        smem_desc(da + ks * 2048, 8192, 1024, kLayoutSW128), idesc_m, true);
            mma_commit(&bar_mma);
        }
        mma_pending = 1;
        ok = mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        mma_phase ^= 1;
        mma_pending = 0;
        tc_fence_after();

        // dU (rows 0..63): fp32 out; -dU as the fp16 operand of MMA-b
        if (lane_row < 64) {
            float v[32];
            tmem_ld32_sync(RDU + lane_base + 32 * wg, v);
            float* dst = dU_all + (item * kChunk + lane_row) * DV + j0 + 32 * wg;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
#pragma unroll
            for (int i8 = 0; i8 < 4; ++i8) {
                __align__(16) __half2 hv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float a = v[8 * i8 + 2 * e], c2 = v[8 * i8 + 2 * e + 1];
                    range_max = fmaxf(range_max, fmaxf(fabsf(a), fabsf(c2)));
                    hv[e] = __floats2half2_rn(-a, -c2);
                }
                *reinterpret_cast<uint4*>(sm + Sm::DU16 + sw128_offset(lane_row, (32 * wg + 8 * i8) * 2)) =
                    *reinterpret_cast<const uint4*>(hv);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // MMA-b: S_acc += Q~^T D + W^T (-dU)
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc_m = instr_desc(kFmtF16, 128, kSliceTc, true, true);
            const uint32_t wq = smem_u32(st + K2::WQ), da = smem_u32(st + Sm::D), du = smem_u32(sm + Sm::DU16);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)   // Q~: rows 64..127 of each WQ tile
                mma_f16(SACC, smem_desc(wq + 8192 + ks * 2048, 16384, 1024, kLayoutSW128),
                        smem_desc(da + ks * 2048, 8192, 1024, kLayoutSW128), idesc_m, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)   // W: rows 0..63 of each WQ tile
                mma_f16(SACC, smem_desc(wq + ks * 2048, 16384, 1024, kLayoutSW128),
                        smem_desc(du + ks * 2048, 8192, 1024, kLayoutSW128), idesc_m, true);
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
            issue(n - 2);   // this stage is no longer read
        }
        if (n - 2 >= 0) copies_issued = m + 3;
        // the fp16 copy of dS for the previous chunk
        if (lane_row < DK) {
            float v[32];
            tmem_ld32_sync(SACC + lane_base + 32 * wg, v);
            put_ds16(v);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (aborted) {
        if (tid == 0) flag_error(hdr, kStatusTimeout);
        // let MMAs and copies this CTA issued finish before its memory goes away
        if (mma_pending) (void)mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        for (int j = copies_done; j < copies_issued; ++j)
            (void)mbar_wait_cycles(&bar_full[(nch - 1 - j) & 1], (j >> 1) & 1, kWaitCycles / 8);
    } else if (d_initial_state && lane_row < DK) {
        float v[32];
        tmem_ld32_sync(SACC + lane_base + 32 * wg, v);
        float* dst = d_initial_state + state_off + (size_t)lane_row * DV + j0 + 32 * wg;
#pragma unroll
        for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    }
    if (range_max > kF16Limit) flag_error(hdr, kStatusRange);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

// ------------------------------------------- backward value-side (bf16) ----
// The backward's products over the value dimension on the tensor cores (bf16
// inputs), one (chunk, head) at a time per CTA:
//     [W; Q~] S -> U = U0 - W S          [D; -dU] S^T -> [dQ~; dW]
//     [U; *] dS'^T -> dK^                 [D; -dU] U^T -> dP (lower)
// and dgamma = rowsum(dS' * S).  S, dS', dU (fp32) are converted to fp16
// 128-byte-swizzled tiles, D = c dO is TMA-loaded (bf16) and converted in
// place, W, Q~, U0 are the forward's fp16 record tiles; the products are
// fp32 in TMEM and go out in fp32 (VSide layout).
template <int DK, int DV>
struct VsSmem {
    static constexpr uint32_t NJ = DV / 64;                       // 64-column value blocks
    static constexpr uint32_t AB = 0;                             // [D; -dU]: NJ tiles of 128 rows
    static constexpr uint32_t S16 = AB + NJ * 16384;              // S: NJ tiles of DK rows (key channel)
    static constexpr uint32_t DS16 = S16 + NJ * DK * 128;         // dS': same
    static constexpr uint32_t U16 = DS16 + NJ * DK * 128;         // U: NJ tiles of 64 rows (+ one spare tile)
    static constexpr uint32_t WQ = U16 + NJ * 8192 + 8192;        // record tiles [W; Q~]
    static constexpr uint32_t U0 = WQ + (DK / 64) * 16384;        // record tiles U0
    static constexpr uint32_t END = U0 + NJ * 8192;
    static constexpr uint32_t TX_BYTES = (DK / 64) * 16384 + NJ * 8192 + NJ * 8192;
    static_assert(END + 1024 <= 232448, "shared memory");
};

template <int DK, int DV>
__global__ void __launch_bounds__(256, 1)
bwd_vside_tc_kernel(const __grid_constant__ CUtensorMap tm_do, ChunkMap map, WsHeader* hdr,
                    const unsigned char* __restrict__ records, const float* __restrict__ states,
                    const float* __restrict__ dS_end, const float* __restrict__ dU_all,
                    float* __restrict__ vside, int H, size_t max_chunks, float scale)
{
    using Sm = VsSmem<DK, DV>;
    using R = TcRec<DK, DV>;
    using VS = VSide<DK>;
    constexpr int NJ = DV / 64;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar_load, bar_mma;
    __shared__ uint32_t s_tmem;
    __shared__ float s_dgam[DK];

    if (hdr->status != kStatusOk) return;
    const int total = hdr->num_chunks * H;
    if ((int)blockIdx.x >= total) return;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int lane_row = (warp & 3) * 32 + (tid & 31);   // TMEM lane = MMA row
    const int wg = warp >> 2;
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
    const uint32_t TA = tmem;                 // [W S; Q~ S]: DV columns
    const uint32_t TB = tmem + DV;            // [dQ~; dW]: DK columns
    const uint32_t TC = tmem + DV + DK;       // [dK^; *]: DK columns
    const uint32_t TD = tmem + DV + 2 * DK;   // [dP; *]: 64 columns
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    float range_max = 0.f;
    uint32_t load_phase = 0, mma_phase = 0;
    bool aborted = false;
    int mma_pending = 0;

    // an item's S, dS' (DK x DV) and dU (64 x DV) in fp32, 8 columns per thread and
    // step; the next item's are loaded into registers while this item's last
    // products and write-out run
    constexpr int NSD = DK * DV / 8 / 256, NU = kChunk * DV / 8 / 256;
    static_assert(DK * DV / 8 % 256 == 0 && kChunk * DV / 8 % 256 == 0, "whole steps");
    float4 rs[2 * NSD], rd[2 * NSD], ru[2 * NU];
    auto load_item = [&](int x) {
        const int c = x / H, hh = x - c * H;
        const size_t it = (size_t)hh * max_chunks + c;
        const float* Sn = states + it * DK * DV;
        const float* dSe = dS_end + it * DK * DV;
        const float* dUc = dU_all + it * kChunk * DV;
#pragma unroll
        for (int j = 0; j < NSD; ++j) {
            const int idx = tid + 256 * j, ch = idx / (DV / 8), j8 = (idx - ch * (DV / 8)) * 8;
            rs[2 * j] = *reinterpret_cast<const float4*>(Sn + (size_t)ch * DV + j8);
            rs[2 * j + 1] = *reinterpret_cast<const float4*>(Sn + (size_t)ch * DV + j8 + 4);
            rd[2 * j] = *reinterpret_cast<const float4*>(dSe + (size_t)ch * DV + j8);
            rd[2 * j + 1] = *reinterpret_cast<const float4*>(dSe + (size_t)ch * DV + j8 + 4);
        }
#pragma unroll
        for (int j = 0; j < NU; ++j) {
            const int idx = tid + 256 * j, r = idx / (DV / 8), j8 = (idx - r * (DV / 8)) * 8;
            ru[2 * j] = *reinterpret_cast<const float4*>(dUc + (size_t)r * DV + j8);
            ru[2 * j + 1] = *reinterpret_cast<const float4*>(dUc + (size_t)r * DV + j8 + 4);
        }
    };
    auto issue_tiles = [&](int x) {   // one thread: item x's record tiles and d_o
        const int c = x / H, hh = x - c * H;
        int s_, t0, l_;
        map.locate(c, s_, t0, l_);
        const unsigned char* rec = records + ((size_t)hh * max_chunks + c) * R::BYTES;
        mbar_arrive_expect_tx(&bar_load, Sm::TX_BYTES);
        bulk_load(sm + Sm::WQ, rec + R::WQ, R::WQ_BYTES, &bar_load);
        bulk_load(sm + Sm::U0, rec + R::U0, R::U0_BYTES, &bar_load);
#pragma unroll
        for (int b = 0; b < NJ; ++b) tma_load_3d(sm + Sm::AB + b * 16384, &tm_do, &bar_load, b * 64, hh, t0);
    };
    int w = blockIdx.x;
    if (tid == 0) issue_tiles(w);
    bool load_pending = true;
    load_item(w);

    while (w < total) {
        const int c = w / H, h = w - c * H;
        int seq, tok0, L;
        map.locate(c, seq, tok0, L);
        const size_t it = (size_t)h * max_chunks + c;
        float* out = vside + it * VS::FLOATS;
        const int nw = w + gridDim.x;

        if (tid < DK) s_dgam[tid] = 0.f;
        __syncthreads();
        // fp16 operands: S and dS' (rows = key channel), -dU (rows 64..127 of [D; -dU]); dgamma
        // DV / 8 consecutive threads share a key row: their dgamma parts are
        // summed by shuffles, then added once (DV / 8 divides 32)
        static_assert(32 % (DV / 8) == 0, "row groups within a warp");
#pragma unroll
        for (int j = 0; j < NSD; ++j) {
            const int idx = tid + 256 * j, ch = idx / (DV / 8), j8 = (idx - ch * (DV / 8)) * 8;
            const float4 s0 = rs[2 * j], s1 = rs[2 * j + 1], d0 = rd[2 * j], d1 = rd[2 * j + 1];
            float gpart = s0.x * d0.x + s0.y * d0.y + s0.z * d0.z + s0.w * d0.w +
                          s1.x * d1.x + s1.y * d1.y + s1.z * d1.z + s1.w * d1.w;
#pragma unroll
            for (int off = DV / 16; off; off >>= 1) gpart += __shfl_xor_sync(0xffffffffu, gpart, off);
            if ((tid & (DV / 8 - 1)) == 0) atomicAdd(&s_dgam[ch], gpart);
            __align__(16) __half2 hs[4] = {__floats2half2_rn(s0.x, s0.y), __floats2half2_rn(s0.z, s0.w),
                                           __floats2half2_rn(s1.x, s1.y), __floats2half2_rn(s1.z, s1.w)};
            __align__(16) __half2 hd[4] = {__floats2half2_rn(d0.x, d0.y), __floats2half2_rn(d0.z, d0.w),
                                           __floats2half2_rn(d1.x, d1.y), __floats2half2_rn(d1.z, d1.w)};
            range_max = fmaxf(range_max, fmaxf(fmaxf(fabsf(s0.x), fabsf(s0.y)), fmaxf(fabsf(s0.z), fabsf(s0.w))));
            range_max = fmaxf(range_max, fmaxf(fmaxf(fabsf(s1.x), fabsf(s1.y)), fmaxf(fabsf(s1.z), fabsf(s1.w))));
            range_max = fmaxf(range_max, fmaxf(fmaxf(fabsf(d0.x), fabsf(d0.y)), fmaxf(fabsf(d0.z), fabsf(d0.w))));
            range_max = fmaxf(range_max, fmaxf(fmaxf(fabsf(d1.x), fabsf(d1.y)), fmaxf(fabsf(d1.z), fabsf(d1.w))));
            const uint32_t o = (j8 >> 6) * (DK * 128) + sw128_offset(ch, (j8 & 63) * 2);
            *reinterpret_cast<uint4*>(sm + Sm::S16 + o) = *reinterpret_cast<const uint4*>(hs);
            *reinterpret_cast<uint4*>(sm + Sm::DS16 + o) = *reinterpret_cast<const uint4*>(hd);
        }
#pragma unroll
        for (int j = 0; j < NU; ++j) {
            const int idx = tid + 256 * j, r = idx / (DV / 8), j8 = (idx - r * (DV / 8)) * 8;
            const float4 u0 = ru[2 * j], u1 = ru[2 * j + 1];
            __align__(16) __half2 hu[4] = {__floats2half2_rn(-u0.x, -u0.y), __floats2half2_rn(-u0.z, -u0.w),
                                           __floats2half2_rn(-u1.x, -u1.y), __floats2half2_rn(-u1.z, -u1.w)};
            range_max = fmaxf(range_max, fmaxf(fmaxf(fabsf(u0.x), fabsf(u0.y)), fmaxf(fabsf(u0.z), fabsf(u0.w))));
            range_max = fmaxf(range_max, fmaxf(fmaxf(fabsf(u1.x), fabsf(u1.y)), fmaxf(fabsf(u1.z), fabsf(u1.w))));
            *reinterpret_cast<uint4*>(sm + Sm::AB + (j8 >> 6) * 16384 + sw128_offset(64 + r, (j8 & 63) * 2)) =
                *reinterpret_cast<const uint4*>(hu);
        }
        // D = c dO: bf16 -> fp16 in place (rows 0..63 of [D; -dU]); rows past the chunk are zero
        const bool ok_load = mbar_wait_cycles(&bar_load, load_phase, kWaitCycles);
        if (__syncthreads_or(!ok_load)) { aborted = true; break; }
        load_phase ^= 1;
        load_pending = false;
        for (int idx = tid; idx < kChunk * DV / 8; idx += 256) {
            const int r = idx / (DV / 8), j8 = (idx - r * (DV / 8)) * 8;
            const uint32_t o = Sm::AB + (j8 >> 6) * 16384 + sw128_offset(r, (j8 & 63) * 2);
            uint4 raw = *reinterpret_cast<const uint4*>(sm + o);
            if (r >= L) raw = make_uint4(0, 0, 0, 0);
            const __nv_bfloat162* db = reinterpret_cast<const __nv_bfloat162*>(&raw);
            __align__(16) __half2 dh[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 x = __bfloat1622float2(db[e]);
                range_max = fmaxf(range_max, fmaxf(fabsf(scale * x.x), fabsf(scale * x.y)));
                dh[e] = __floats2half2_rn(scale * x.x, scale * x.y);
            }
            *reinterpret_cast<uint4*>(sm + o) = *reinterpret_cast<const uint4*>(dh);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // [W; Q~] S -> TA and [D; -dU] S^T -> TB
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc_a = instr_desc(kFmtF16, 128, DV, false, true);   // B MN-major
            constexpr uint32_t idesc_b = instr_desc(kFmtF16, 128, DK, false, false);  // both K-major
            const uint32_t wq = smem_u32(sm + Sm::WQ), s16 = smem_u32(sm + Sm::S16), ab = smem_u32(sm + Sm::AB);
#pragma unroll
            for (int kb = 0; kb < DK / 64; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(TA, smem_desc(wq + kb * 16384 + ks * 32, 16, 1024, kLayoutSW128),
                            smem_desc(s16 + kb * 8192 + ks * 2048, DK * 128, 1024, kLayoutSW128), idesc_a,
                            (kb | ks) != 0);
#pragma unroll
            for (int kb = 0; kb < NJ; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(TB, smem_desc(ab + kb * 16384 + ks * 32, 16, 1024, kLayoutSW128),
                            smem_desc(s16 + kb * (DK * 128) + ks * 32, 16, 1024, kLayoutSW128), idesc_b,
                            (kb | ks) != 0);
            mma_commit(&bar_mma);
        }
        mma_pending = 1;
        bool ok = mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        mma_phase ^= 1;
        mma_pending = 0;
        tc_fence_after();

        // U = U0 - W S (rows 0..63) -> fp16 U tiles
        if (lane_row < 64) {
#pragma unroll 1
            for (int cb = wg; cb < DV / 32; cb += 2) {
                float v[32];
                tmem_ld32_sync(TA + lane_base + 32 * cb, v);
#pragma unroll
                for (int i8 = 0; i8 < 4; ++i8) {
                    const int col = 32 * cb + 8 * i8;
                    const uint32_t o = (col >> 6) * 8192 + sw128_offset(lane_row, (col & 63) * 2);
                    const uint4 u0raw = *reinterpret_cast<const uint4*>(sm + Sm::U0 + o);
                    const __half2* u0 = reinterpret_cast<const __half2*>(&u0raw);
                    __align__(16) __half2 hv[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 u0f = __half22float2(u0[e]);
                        const float a = u0f.x - v[8 * i8 + 2 * e], b2 = u0f.y - v[8 * i8 + 2 * e + 1];
                        range_max = fmaxf(range_max, fmaxf(fabsf(a), fabsf(b2)));
                        hv[e] = __floats2half2_rn(a, b2);
                    }
                    *reinterpret_cast<uint4*>(sm + Sm::U16 + o) = *reinterpret_cast<const uint4*>(hv);
                }
            }
        }
        // [dQ~; dW] out (all 128 lanes)
#pragma unroll 1
        for (int cb = wg; cb < DK / 32; cb += 2) {
            float v[32];
            tmem_ld32_sync(TB + lane_base + 32 * cb, v);
            float* dst = lane_row < 64 ? out + VS::DQT + (size_t)lane_row * DK + 32 * cb
                                       : out + VS::DW + (size_t)(lane_row - 64) * DK + 32 * cb;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // [U; *] dS'^T -> TC and [D; -dU] U^T -> TD
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc_c = instr_desc(kFmtF16, 128, DK, false, false);
            constexpr uint32_t idesc_d = instr_desc(kFmtF16, 128, 64, false, false);
            const uint32_t u16 = smem_u32(sm + Sm::U16), ds16 = smem_u32(sm + Sm::DS16), ab = smem_u32(sm + Sm::AB);
#pragma unroll
            for (int kb = 0; kb < NJ; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(TC, smem_desc(u16 + kb * 8192 + ks * 32, 16, 1024, kLayoutSW128),
                            smem_desc(ds16 + kb * (DK * 128) + ks * 32, 16, 1024, kLayoutSW128), idesc_c,
                            (kb | ks) != 0);
#pragma unroll
            for (int kb = 0; kb < NJ; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(TD, smem_desc(ab + kb * 16384 + ks * 32, 16, 1024, kLayoutSW128),
                            smem_desc(u16 + kb * 8192 + ks * 32, 16, 1024, kLayoutSW128), idesc_d,
                            (kb | ks) != 0);
            mma_commit(&bar_mma);
        }
        mma_pending = 1;
        if (nw < total) load_item(nw);   // in flight across these MMAs and the write-out below
        ok = mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        mma_phase ^= 1;
        mma_pending = 0;
        tc_fence_after();
        // every operand buffer is read: the next item's record tiles and d_o come in
        if (nw < total) {
            if (tid == 0) issue_tiles(nw);
            load_pending = true;
        }

        // dK^ and dP (rows 0..63) out; dgamma
        if (lane_row < 64) {
#pragma unroll 1
            for (int cb = wg; cb < DK / 32; cb += 2) {
                float v[32];
                tmem_ld32_sync(TC + lane_base + 32 * cb, v);
                float* dst = out + VS::DKH + (size_t)lane_row * DK + 32 * cb;
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
            }
            {
                float v[32];
                tmem_ld32_sync(TD + lane_base + 32 * wg, v);
                float* dst = out + VS::DP + (size_t)lane_row * kChunk + 32 * wg;
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    const int col = 32 * wg + i;
                    *reinterpret_cast<float4*>(dst + i) =
                        make_float4(col <= lane_row ? v[i] : 0.f, col + 1 <= lane_row ? v[i + 1] : 0.f,
                                    col + 2 <= lane_row ? v[i + 2] : 0.f, col + 3 <= lane_row ? v[i + 3] : 0.f);
                }
            }
        }
        if (tid < DK) out[VS::DGAM + tid] = s_dgam[tid];
        tc_fence_before();
        __syncthreads();   // smem and TMEM are free for the next item
        w = nw;
    }

    if (aborted) {
        if (tid == 0) flag_error(hdr, kStatusTimeout);
        if (mma_pending) (void)mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        if (load_pending) (void)mbar_wait_cycles(&bar_load, load_phase, kWaitCycles / 4);
    }
    if (range_max > kF16Limit) flag_error(hdr, kStatusRange);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------ backward T-chain (bf16) ----
// The products of the backward through W = T diag(beta) K~, U0 = T diag(beta) V
// and T = (I + A)^{-1} on the tensor cores (bf16 inputs), one (chunk, head) at
// a time per CTA:
//     [Z | Y] = T^T [dU | dW]          -> dv = beta Z, dK~ = beta Y, dbeta parts <Z, v> + <Y, K~>
//     dT = (dW K~^T + dU V^T) diag(beta) -> X1 = dT T^T -> dA = -T^T X1 (strictly lower)
// T, K~, V are the forward kernel's fp16 tiles (backward mode), dU and dW
// (fp32) are converted to fp16; products accumulate in fp32 in TMEM.
template <int DK, int DV>
struct TchSmem {
    // fp16 128-byte-swizzled tiles of 64 rows x 64 columns (8 KB); an operand read
    // as a 128-row MMA operand is followed by another valid tile
    static constexpr uint32_t T = 0;                        // T [i][r]
    static constexpr uint32_t X1 = T + 8192;                // X1 [j][i]
    static constexpr uint32_t DU = X1 + 8192;               // dU [r][j]: DV / 64 tiles
    static constexpr uint32_t DW = DU + (DV / 64) * 8192;   // dW [r][c]: DK / 64 tiles
    static constexpr uint32_t DT = DW + (DK / 64) * 8192;   // dT diag(beta) [r][i], then a spare tile
    static constexpr uint32_t KT = DT + 16384;              // K~ [i][c]: DK / 64 tiles
    static constexpr uint32_t V = KT + (DK / 64) * 8192;    // V [i][j]: DV / 64 tiles
    static constexpr uint32_t END = V + (DV / 64) * 8192;
};

template <int DK, int DV>
__global__ void __launch_bounds__(256, 1)
bwd_tchain_tc_kernel(ChunkMap map, WsHeader* hdr, const unsigned char* __restrict__ tiles,
                     const float* __restrict__ dU_all, const float* __restrict__ beta,
                     float* __restrict__ vside, __nv_bfloat16* __restrict__ dv, int H, size_t max_chunks)
{
    using Sm = TchSmem<DK, DV>;
    using BT = BwdTiles<DK, DV>;
    using VS = VSide<DK>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar_load, bar_mma;
    __shared__ uint32_t s_tmem;
    __shared__ float s_beta[kChunk], s_dbp[kChunk];

    if (hdr->status != kStatusOk) return;
    const int total = hdr->num_chunks * H;
    if ((int)blockIdx.x >= total) return;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int lane_row = (warp & 3) * 32 + (tid & 31);   // TMEM lane = MMA row
    const int wg = warp >> 2;
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
    const uint32_t TZY = tmem;                   // [Z | Y]: DV + DK columns
    const uint32_t TDT = tmem + DV + DK;         // dT: 64
    const uint32_t TX1 = TDT + 64;               // X1: 64
    const uint32_t TDA = TX1 + 64;               // T^T X1: 64
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    float range_max = 0.f;
    uint32_t load_phase = 0, mma_phase = 0;
    bool aborted = false;
    int mma_pending = 0;

    auto mma_wait = [&]() -> bool {
        mma_pending = 1;
        const bool ok = mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        if (ok) {
            mma_phase ^= 1;
            mma_pending = 0;
        }
        return ok;
    };
    // fp16 copy of 8 fp32 values into a swizzled tile row
    auto put8 = [&](uint32_t off, const float4& a, const float4& b, float sgn) {
        __align__(16) __half2 hv[4] = {__floats2half2_rn(sgn * a.x, sgn * a.y), __floats2half2_rn(sgn * a.z, sgn * a.w),
                                       __floats2half2_rn(sgn * b.x, sgn * b.y), __floats2half2_rn(sgn * b.z, sgn * b.w)};
        range_max = fmaxf(range_max, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))));
        range_max = fmaxf(range_max, fmaxf(fmaxf(fabsf(b.x), fabsf(b.y)), fmaxf(fabsf(b.z), fabsf(b.w))));
        *reinterpret_cast<uint4*>(sm + off) = *reinterpret_cast<const uint4*>(hv);
    };

    // an item's dU (64 x DV) and dW (64 x DK) in fp32, 8 columns per thread and
    // step; the next item's are loaded into registers while this item's
    // write-out and last products run
    constexpr int NUJ = kChunk * DV / 8 / 256, NWJ = kChunk * DK / 8 / 256;
    static_assert(kChunk * DV / 8 % 256 == 0 && kChunk * DK / 8 % 256 == 0, "whole steps");
    float4 ru[2 * NUJ], rw[2 * NWJ];
    auto load_item = [&](int x) {
        const int c = x / H, hh = x - c * H;
        const size_t it = (size_t)hh * max_chunks + c;
        const float* dUc = dU_all + it * kChunk * DV;
        const float* dWc = vside + it * VS::FLOATS + VS::DW;
#pragma unroll
        for (int j = 0; j < NUJ; ++j) {
            const int idx = tid + 256 * j, r = idx / (DV / 8), j8 = (idx - r * (DV / 8)) * 8;
            ru[2 * j] = *reinterpret_cast<const float4*>(dUc + (size_t)r * DV + j8);
            ru[2 * j + 1] = *reinterpret_cast<const float4*>(dUc + (size_t)r * DV + j8 + 4);
        }
#pragma unroll
        for (int j = 0; j < NWJ; ++j) {
            const int idx = tid + 256 * j, r = idx / (DK / 8), c8 = (idx - r * (DK / 8)) * 8;
            rw[2 * j] = *reinterpret_cast<const float4*>(dWc + (size_t)r * DK + c8);
            rw[2 * j + 1] = *reinterpret_cast<const float4*>(dWc + (size_t)r * DK + c8 + 4);
        }
    };
    auto issue_tiles = [&](int x) {   // one thread: item x's fp16 T, K~, V tiles
        const int c = x / H, hh = x - c * H;
        const unsigned char* tl = tiles + ((size_t)hh * max_chunks + c) * BT::BYTES;
        mbar_arrive_expect_tx(&bar_load, BT::TILE_BYTES);
        bulk_load(sm + Sm::T, tl + BT::T, 8192, &bar_load);
        bulk_load(sm + Sm::KT, tl + BT::KT, (DK / 64) * 8192, &bar_load);
        bulk_load(sm + Sm::V, tl + BT::V, (DV / 64) * 8192, &bar_load);
    };
    int w = blockIdx.x;
    if (tid == 0) issue_tiles(w);
    bool load_pending = true;
    load_item(w);

    while (w < total) {
        const int c = w / H, h = w - c * H;
        int seq, tok0, L;
        map.locate(c, seq, tok0, L);
        const size_t it = (size_t)h * max_chunks + c;
        float* out = vside + it * VS::FLOATS;
        const int nw = w + gridDim.x;

        if (tid < kChunk) {
            s_beta[tid] = tid < L ? beta[(size_t)(tok0 + tid) * H + h] : 0.f;
            s_dbp[tid] = 0.f;
        }
        // dU and dW (rows = token) as fp16 tiles
#pragma unroll
        for (int j = 0; j < NUJ; ++j) {
            const int idx = tid + 256 * j, r = idx / (DV / 8), j8 = (idx - r * (DV / 8)) * 8;
            put8(Sm::DU + (j8 >> 6) * 8192 + sw128_offset(r, (j8 & 63) * 2), ru[2 * j], ru[2 * j + 1], 1.f);
        }
#pragma unroll
        for (int j = 0; j < NWJ; ++j) {
            const int idx = tid + 256 * j, r = idx / (DK / 8), c8 = (idx - r * (DK / 8)) * 8;
            put8(Sm::DW + (c8 >> 6) * 8192 + sw128_offset(r, (c8 & 63) * 2), rw[2 * j], rw[2 * j + 1], 1.f);
        }
        const bool ok_load = mbar_wait_cycles(&bar_load, load_phase, kWaitCycles);
        fence_proxy_async_smem();
        tc_fence_before();
        if (__syncthreads_or(!ok_load)) { aborted = true; break; }
        load_phase ^= 1;
        load_pending = false;

        // [Z | Y] = T^T [dU | dW];  dT_raw = dW K~^T + dU V^T
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc_zy = instr_desc(kFmtF16, 128, DV + DK, true, true);   // A, B MN-major
            constexpr uint32_t idesc_dt = instr_desc(kFmtF16, 128, 64, false, false);     // both K-major
            const uint32_t t = smem_u32(sm + Sm::T), du = smem_u32(sm + Sm::DU), dw = smem_u32(sm + Sm::DW);
            const uint32_t kt = smem_u32(sm + Sm::KT), vv = smem_u32(sm + Sm::V);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_f16(TZY, smem_desc(t + ks * 2048, 8192, 1024, kLayoutSW128),
                        smem_desc(du + ks * 2048, 8192, 1024, kLayoutSW128), idesc_zy, ks != 0);
#pragma unroll
            for (int b = 0; b < DK / 64; ++b)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(TDT, smem_desc(dw + b * 8192 + ks * 32, 16, 1024, kLayoutSW128),
                            smem_desc(kt + b * 8192 + ks * 32, 16, 1024, kLayoutSW128), idesc_dt, (b | ks) != 0);
#pragma unroll
            for (int b = 0; b < DV / 64; ++b)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(TDT, smem_desc(du + b * 8192 + ks * 32, 16, 1024, kLayoutSW128),
                            smem_desc(vv + b * 8192 + ks * 32, 16, 1024, kLayoutSW128), idesc_dt, true);
            mma_commit(&bar_mma);
        }
        bool ok = mma_wait();
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        tc_fence_after();

        // dT diag(beta) -> fp16 tile (rows 0..63)
        if (lane_row < 64) {
            float v[32];
            tmem_ld32_sync(TDT + lane_base + 32 * wg, v);
#pragma unroll
            for (int i8 = 0; i8 < 4; ++i8) {
                const int col = 32 * wg + 8 * i8;
                const float4 a = make_float4(v[8 * i8] * s_beta[col], v[8 * i8 + 1] * s_beta[col + 1],
                                             v[8 * i8 + 2] * s_beta[col + 2], v[8 * i8 + 3] * s_beta[col + 3]);
                const float4 b = make_float4(v[8 * i8 + 4] * s_beta[col + 4], v[8 * i8 + 5] * s_beta[col + 5],
                                             v[8 * i8 + 6] * s_beta[col + 6], v[8 * i8 + 7] * s_beta[col + 7]);
                put8(Sm::DT + sw128_offset(lane_row, col * 2), a, b, 1.f);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // X1 = dT T^T
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc = instr_desc(kFmtF16, 128, 64, false, false);
            const uint32_t dt = smem_u32(sm + Sm::DT), t = smem_u32(sm + Sm::T);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_f16(TX1, smem_desc(dt + ks * 32, 16, 1024, kLayoutSW128),
                        smem_desc(t + ks * 32, 16, 1024, kLayoutSW128), idesc, ks != 0);
            mma_commit(&bar_mma);
        }
        if (nw < total) load_item(nw);   // in flight across the rest of this item
        // meanwhile: dv = beta Z (out), dK~ = beta Y (out), dbeta parts <Z, v> + <Y, K~>
        if (lane_row < 64) {
            const int r = lane_row;
            const float br = s_beta[r];
            float part = 0.f;
#pragma unroll 1
            for (int cb = wg; cb < (DV + DK) / 32; cb += 2) {
                float v[32];
                tmem_ld32_sync(TZY + lane_base + 32 * cb, v);
                const bool zpart = 32 * cb < DV;
                const int col0 = zpart ? 32 * cb : 32 * cb - DV;
                const uint32_t base = zpart ? Sm::V : Sm::KT;
#pragma unroll
                for (int i8 = 0; i8 < 4; ++i8) {
                    const int col = col0 + 8 * i8;
                    const uint4 raw = *reinterpret_cast<const uint4*>(sm + base + (col >> 6) * 8192 + sw128_offset(r, (col & 63) * 2));
                    const __half2* hp = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __half22float2(hp[e]);
                        part += v[8 * i8 + 2 * e] * f.x + v[8 * i8 + 2 * e + 1] * f.y;
                    }
                }
                if (zpart) {
                    if (r < L) {
                        __nv_bfloat16* dst = dv + ((size_t)(tok0 + r) * H + h) * DV + col0;
#pragma unroll
                        for (int i8 = 0; i8 < 4; ++i8) {
                            __align__(16) __nv_bfloat162 bv[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                bv[e] = __floats2bfloat162_rn(br * v[8 * i8 + 2 * e], br * v[8 * i8 + 2 * e + 1]);
                            *reinterpret_cast<uint4*>(dst + 8 * i8) = *reinterpret_cast<const uint4*>(bv);
                        }
                    }
                } else {
                    float* dst = out + VS::DKT + (size_t)r * DK + col0;
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(dst + i) = make_float4(br * v[i], br * v[i + 1], br * v[i + 2], br * v[i + 3]);
                }
            }
            atomicAdd(&s_dbp[r], part);
        }
        ok = mma_wait();
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        tc_fence_after();

        // X1 (rows j) -> fp16 tile [j][i]
        if (lane_row < 64) {
            float v[32];
            tmem_ld32_sync(TX1 + lane_base + 32 * wg, v);
#pragma unroll
            for (int i8 = 0; i8 < 4; ++i8) {
                const float4 a = make_float4(v[8 * i8], v[8 * i8 + 1], v[8 * i8 + 2], v[8 * i8 + 3]);
                const float4 b = make_float4(v[8 * i8 + 4], v[8 * i8 + 5], v[8 * i8 + 6], v[8 * i8 + 7]);
                put8(Sm::X1 + sw128_offset(lane_row, (32 * wg + 8 * i8) * 2), a, b, 1.f);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // T^T X1
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc = instr_desc(kFmtF16, 128, 64, true, true);
            const uint32_t t = smem_u32(sm + Sm::T), x1 = smem_u32(sm + Sm::X1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_f16(TDA, smem_desc(t + ks * 2048, 8192, 1024, kLayoutSW128),
                        smem_desc(x1 + ks * 2048, 8192, 1024, kLayoutSW128), idesc, ks != 0);
            mma_commit(&bar_mma);
        }
        ok = mma_wait();
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        tc_fence_after();
        // every tile is read: the next item's come in
        if (nw < total) {
            if (tid == 0) issue_tiles(nw);
            load_pending = true;
        }
        // dA = -T^T X1, strictly lower (rows 0..63); dbeta parts
        if (lane_row < 64) {
            float v[32];
            tmem_ld32_sync(TDA + lane_base + 32 * wg, v);
            float* dst = out + VS::DA + (size_t)lane_row * kChunk + 32 * wg;
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const int col = 32 * wg + i;
                *reinterpret_cast<float4*>(dst + i) =
                    make_float4(col < lane_row ? -v[i] : 0.f, col + 1 < lane_row ? -v[i + 1] : 0.f,
                                col + 2 < lane_row ? -v[i + 2] : 0.f, col + 3 < lane_row ? -v[i + 3] : 0.f);
            }
        }
        if (tid < kChunk) out[VS::DBP + tid] = s_dbp[tid];
        tc_fence_before();
        __syncthreads();   // smem and TMEM are free for the next item
        w = nw;
    }

    if (aborted) {
        if (tid == 0) flag_error(hdr, kStatusTimeout);
        if (mma_pending) (void)mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        if (load_pending) (void)mbar_wait_cycles(&bar_load, load_phase, kWaitCycles / 4);
    }
    if (range_max > kF16Limit) flag_error(hdr, kStatusRange);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// --------------------------------------- backward split-factor part (bf16) ----
// The rest of the backward for chunks without strong decay, on the tensor
// cores in tf32 (bf16 inputs): with K_l = k e^{g - g_m}, K_r = k e^{g_m - g},
// Q_l = q e^{g - g_m} (fp32 range, hence tf32) and dM = diag(beta) dA,
//     [dK_l^T | dQ_l^T] = K_r^T [dM; dP]^T        dK_r^T = [K_l^T | Q_l^T] [dM^T | dP^T]^T
// so that TMEM lane = key channel; then the decay factors and the suffix sums
// of dlog_alpha per channel, and dbeta = (parts through W, U0) + rowsum(dA M)
// with M from the forward kernel.  Every operand is K-major.
// A CTA takes its items in turn.  The operand buffers are dead from the end of
// an item's MMAs, so the next item's k, q, log_alpha (TMA) and dA, dP (bulk
// copies) are fetched into them then, behind this item's element pass, and an
// item builds its operands from shared memory.  The operand build keeps a copy
// of the item's k and q for its element pass, whose other operands (dK~, dK^,
// dQ~) load into registers while the MMAs run.
template <int DK, int DV>
struct SpSmem {
    static constexpr uint32_t G = 0;                        // g (natural log) [64][DK] fp32, later dg
    static constexpr uint32_t KRT = G + 64 * DK * 4;        // K_r^T [c][i]: 2 tiles (32 i) of DK rows x 128 B
    static constexpr uint32_t KLQT = KRT + 2 * DK * 128;    // [K_l^T | Q_l^T] [c][r]: 4 tiles
    static constexpr uint32_t DMP = KLQT + 4 * DK * 128;    // [dM; dP] [r][i]: 2 tiles of 128 rows x 128 B
    static constexpr uint32_t DMPT = DMP + 2 * 16384;       // [dM^T | dP^T] [i][r]: 4 tiles of 64 rows x 128 B
    static constexpr uint32_t KQ = DMPT + 4 * 8192;         // this item's k, q [64][DK] bf16, for its element pass
    static constexpr uint32_t END = KQ + 2 * 64 * DK * 2;
    // the next item's inputs, each in a buffer that is written only after it has been read
    static constexpr uint32_t PF_LA = KRT;                  // log_alpha [64][DK] fp32
    static constexpr uint32_t PF_K = DMP;                   // k [64][DK] bf16
    static constexpr uint32_t PF_Q = DMP + 64 * DK * 2;     // q [64][DK] bf16
    static constexpr uint32_t PF_DA = DMPT;                 // dA [64][64] fp32
    static constexpr uint32_t PF_DP = DMPT + 64 * 64 * 4;   // dP [64][64] fp32
    static_assert(64 * DK * 4 <= KLQT - KRT && 2 * 64 * DK * 2 <= DMPT - DMP && 2 * 64 * 64 * 4 <= KQ - DMPT,
                  "prefetch buffers");
    static_assert(END + 1024 <= 232448, "shared memory");
};

template <int DK, int DV>
__global__ void __launch_bounds__(256, 1)
bwd_split_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_la, const __nv_bfloat16* __restrict__ q,
                    const __nv_bfloat16* __restrict__ k, const float* __restrict__ log_alpha,
                    const float* __restrict__ beta, ChunkMap map, WsHeader* hdr,
                    const unsigned char* __restrict__ tiles, const int* __restrict__ flags,
                    const float* __restrict__ vside, __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk,
                    float* __restrict__ dla, float* __restrict__ dbeta, int H, size_t max_chunks, int gate)
{
    using Sm = SpSmem<DK, DV>;
    using BT = BwdTiles<DK, DV>;
    using VS = VSide<DK>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar_mma, bar_load;
    __shared__ uint32_t s_tmem;
    __shared__ float s_gm[DK], s_gl[DK], s_dgl[DK], s_beta[kChunk];

    if (hdr->status != kStatusOk) return;
    const int total = hdr->num_chunks * H;
    // this CTA's items are blockIdx.x + j gridDim.x, less the strong-decay chunks
    // (the exact CUDA-core path takes those)
    auto next_item = [&](int x) {
        while (x < total) {
            const int c = x / H;
            if (!flags[(size_t)(x - c * H) * max_chunks + c]) break;
            x += gridDim.x;
        }
        return x;
    };
    int w = next_item(blockIdx.x);
    if (w >= total) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lane_row = (warp & 3) * 32 + (tid & 31);   // TMEM lane = key channel
    const int wg = warp >> 2;                            // tokens [32 wg, 32 wg + 32)
    const size_t rowk = (size_t)H * DK;
    const uint32_t load_bytes = 2 * 64 * DK * 2 + 2 * 64 * 64 * 4 + (gate == kGateChannel ? 64 * DK * 4 : 0);
    auto prefetch = [&](int x) {   // one thread: item x's k, q, log_alpha, dA, dP
        const int c = x / H, hh = x - c * H;
        int s_, t0, l_;
        map.locate(c, s_, t0, l_);
        const float* xv = vside + ((size_t)hh * max_chunks + c) * VS::FLOATS;
        mbar_arrive_expect_tx(&bar_load, load_bytes);
        tma_load_3d(sm + Sm::PF_K, &tm_k, &bar_load, 0, hh, t0);
        tma_load_3d(sm + Sm::PF_Q, &tm_q, &bar_load, 0, hh, t0);
        if (gate == kGateChannel) tma_load_3d(sm + Sm::PF_LA, &tm_la, &bar_load, 0, hh, t0);
        bulk_load(sm + Sm::PF_DA, xv + VS::DA, 64 * 64 * 4, &bar_load);
        bulk_load(sm + Sm::PF_DP, xv + VS::DP, 64 * 64 * 4, &bar_load);
    };
    auto load_beta = [&](int x) {   // threads 128 .. 191: item x's beta of token tid - 128
        const int c = x / H, hh = x - c * H, r = tid - 128;
        int s_, t0, l_;
        map.locate(c, s_, t0, l_);
        return r < l_ ? beta[(size_t)(t0 + r) * H + hh] : 0.f;
    };
    const bool beta_thread = tid >= 128 && tid < 128 + kChunk;
    if (tid == 0) {
        mbar_init(&bar_mma, 1);
        mbar_init(&bar_load, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_q);
        if (gate == kGateChannel) tma_prefetch_desc(&tm_la);
    }
    if (warp == 0) {
        tmem_alloc(&s_tmem, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const uint32_t T1 = tmem;          // [dK_l^T | dQ_l^T]: 128 columns (token r)
    const uint32_t T2 = tmem + 128;    // dK_r^T: 64 columns (token i)
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    if (tid == 0) prefetch(w);
    float bnext = beta_thread ? load_beta(w) : 0.f;
    uint32_t mma_phase = 0, load_phase = 0;
    bool aborted = false, load_pending = true, mma_pending = false;
    float* g = reinterpret_cast<float*>(sm + Sm::G);

    while (w < total) {
        const int c = w / H, h = w - c * H;
        const size_t it = (size_t)h * max_chunks + c;
        int seq, tok0, L;
        map.locate(c, seq, tok0, L);
        const int nw = next_item(w + gridDim.x);
        const float* vs = vside + it * VS::FLOATS;
        const float* Mg = reinterpret_cast<const float*>(tiles + it * BT::BYTES + BT::M);
        if (beta_thread) s_beta[tid - 128] = bnext;
        // this thread's entries of M (used once the MMAs are issued): step j covers
        // column (tid + 256 j) % 64, rows 4 ((tid + 256 j) / 64) + [0, 4), as dA below
        float mm[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int idx = tid + 256 * j, i = idx & 63, r4 = (idx >> 6) * 4;
#pragma unroll
            for (int t = 0; t < 4; ++t) mm[j][t] = Mg[(r4 + t) * kChunk + i];
        }
        const float dbp = tid < kChunk ? vs[VS::DBP + tid] : 0.f;   // dbeta parts through W, U0
        const float dgam = tid < DK ? vs[VS::DGAM + tid] : 0.f;   // for the dlog_alpha scan
        const bool got = mbar_wait_cycles(&bar_load, load_phase, kWaitCycles);
        if (__syncthreads_or(!got)) { aborted = true; break; }
        load_phase ^= 1;
        load_pending = false;

        // cumulative log-decay (natural log) per channel; g_m, g_{L-1}
        if (tid < DK) {
            float acc = 0.f;
            if (gate == kGateChannel) {
                const float* la = reinterpret_cast<const float*>(sm + Sm::PF_LA) + tid;
#pragma unroll 16
                for (int r = 0; r < kChunk; ++r) {
                    acc += (r < L) ? la[r * DK] : 0.f;
                    g[r * DK + tid] = acc;
                }
            } else if (gate == kGateHead) {
                const float* la = log_alpha + (size_t)tok0 * H + h;
#pragma unroll 16   // the loads are independent: keep 16 in flight
                for (int r = 0; r < kChunk; ++r) {
                    acc += (r < L) ? la[(size_t)r * H] : 0.f;
                    g[r * DK + tid] = acc;
                }
            } else {
                for (int r = 0; r < kChunk; ++r) g[r * DK + tid] = 0.f;
            }
            s_gm[tid] = g[((L - 1) >> 1) * DK + tid];
            s_gl[tid] = g[(L - 1) * DK + tid];
            s_dgl[tid] = 0.f;
        }
        // dA, dP by column: step j holds column idx % 64, rows 4 (idx / 64) + [0, 4)
        // (idx = tid + 256 j), so that both [dM; dP] (row-major: a warp fills one
        // row segment) and its transpose (a warp fills one 16-byte chunk of 32
        // rows) are stored without bank conflicts
        float da[4][4], dp[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int idx = tid + 256 * j, i = idx & 63, r4 = (idx >> 6) * 4;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                da[j][t] = reinterpret_cast<const float*>(sm + Sm::PF_DA)[(r4 + t) * 64 + i];
                dp[j][t] = reinterpret_cast<const float*>(sm + Sm::PF_DP)[(r4 + t) * 64 + i];
            }
        }
        __syncthreads();

        // tf32 operands.  K_r^T, K_l^T, Q_l^T: (channel, 4 tokens) per step
        {
            const __nv_bfloat16* pk = reinterpret_cast<const __nv_bfloat16*>(sm + Sm::PF_K);
            const __nv_bfloat16* pq = reinterpret_cast<const __nv_bfloat16*>(sm + Sm::PF_Q);
            __nv_bfloat16* kq = reinterpret_cast<__nv_bfloat16*>(sm + Sm::KQ);   // k rows, then q rows
            const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
#pragma unroll
            for (int idx = tid; idx < DK * (kChunk / 4); idx += 256) {
                const int ch = idx % DK, r4 = (idx / DK) * 4;
                float kr[4], kl[4], ql[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int r = r4 + t;
                    const __nv_bfloat16 kb = r < L ? pk[r * DK + ch] : zero, qb = r < L ? pq[r * DK + ch] : zero;
                    kq[r * DK + ch] = kb;
                    kq[(kChunk + r) * DK + ch] = qb;
                    const float kk = __bfloat162float(kb), qq = __bfloat162float(qb);
                    const float d = g[r * DK + ch] - s_gm[ch];
                    const float fl = __expf(d), fr = __expf(-d);
                    kr[t] = round_tf32_alu(kk * fr);
                    kl[t] = round_tf32_alu(kk * fl);
                    ql[t] = round_tf32_alu(qq * fl);
                }
                *reinterpret_cast<float4*>(sm + Sm::KRT + f_off(ch, r4, DK * 128)) = make_float4(kr[0], kr[1], kr[2], kr[3]);
                *reinterpret_cast<float4*>(sm + Sm::KLQT + f_off(ch, r4, DK * 128)) = make_float4(kl[0], kl[1], kl[2], kl[3]);
                *reinterpret_cast<float4*>(sm + Sm::KLQT + f_off(ch, 64 + r4, DK * 128)) = make_float4(ql[0], ql[1], ql[2], ql[3]);
            }
        }
        __syncthreads();   // k, q (under [dM; dP]) and dA, dP (under its transpose) are read
        // [dM; dP] and their transposes
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int idx = tid + 256 * j, i = idx & 63, r4 = (idx >> 6) * 4;
            float dm[4], pp[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                dm[t] = round_tf32_alu(s_beta[r4 + t] * da[j][t]);
                pp[t] = round_tf32_alu(dp[j][t]);
                *reinterpret_cast<float*>(sm + Sm::DMP + f_off(r4 + t, i, 16384)) = dm[t];
                *reinterpret_cast<float*>(sm + Sm::DMP + f_off(64 + r4 + t, i, 16384)) = pp[t];
            }
            *reinterpret_cast<float4*>(sm + Sm::DMPT + f_off(i, r4, 8192)) = make_float4(dm[0], dm[1], dm[2], dm[3]);
            *reinterpret_cast<float4*>(sm + Sm::DMPT + f_off(i, 64 + r4, 8192)) = make_float4(pp[0], pp[1], pp[2], pp[3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc1 = instr_desc(kFmtTF32, 128, 128);
            constexpr uint32_t idesc2 = instr_desc(kFmtTF32, 128, 64);
            const uint32_t krt = smem_u32(sm + Sm::KRT), klqt = smem_u32(sm + Sm::KLQT);
            const uint32_t dmp = smem_u32(sm + Sm::DMP), dmpt = smem_u32(sm + Sm::DMPT);
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_tf32(T1, smem_desc(krt + kb * (DK * 128) + ks * 32, 16, 1024, kLayoutSW128),
                             smem_desc(dmp + kb * 16384 + ks * 32, 16, 1024, kLayoutSW128), idesc1, (kb | ks) != 0);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_tf32(T2, smem_desc(klqt + kb * (DK * 128) + ks * 32, 16, 1024, kLayoutSW128),
                             smem_desc(dmpt + kb * 8192 + ks * 32, 16, 1024, kLayoutSW128), idesc2, (kb | ks) != 0);
            mma_commit(&bar_mma);
        }
        mma_pending = true;
        // this thread's element-pass operands from global memory (channel lane_row,
        // tokens [32 wg, 32 wg + 32)), in flight across the MMAs
        float dqtv[32], dktv[32], dkhv[32];
        if (lane_row < DK) {
#pragma unroll
            for (int t = 0; t < 32; ++t) {
                const int r = 32 * wg + t;
                dqtv[t] = vs[VS::DQT + r * DK + lane_row];
                dktv[t] = vs[VS::DKT + r * DK + lane_row];
                dkhv[t] = vs[VS::DKH + r * DK + lane_row];
            }
        }
        // meanwhile: rowsum(dA M) for dbeta over this warp's 32 columns of 4 rows per
        // step (the other 32 columns are in the neighbouring warp)
        float rs[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int t = 0; t < 4; ++t) rs[j][t] = da[j][t] * mm[j][t];
#pragma unroll
            for (int off = 16; off; off >>= 1)
#pragma unroll
                for (int t = 0; t < 4; ++t) rs[j][t] += __shfl_xor_sync(0xffffffffu, rs[j][t], off);
        }
        const bool ok = mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        mma_phase ^= 1;
        mma_pending = false;
        tc_fence_after();
        // the operand buffers are free: the next item's inputs land behind the element pass
        if (nw < total) {
            if (tid == 0) prefetch(nw);
            load_pending = true;
            if (beta_thread) bnext = load_beta(nw);
        }
        // the row sums' two column halves, in [K_l^T | Q_l^T]'s space (read by the
        // MMAs, not a prefetch target): [2][64]
        float* rowsum = reinterpret_cast<float*>(sm + Sm::KLQT);
        if (lane == 0) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int t = 0; t < 4; ++t) rowsum[(warp & 1) * kChunk + ((tid + 256 * j) >> 6) * 4 + t] = rs[j][t];
        }

        // dq, dk and dg for channel lane_row, tokens [32 wg, 32 wg + 32)
        const __nv_bfloat16* kq = reinterpret_cast<const __nv_bfloat16*>(sm + Sm::KQ);
        if (lane_row < DK) {
            const int ch = lane_row;
            const float gm = s_gm[ch], gl = s_gl[ch];
            const float egm = __expf(gm), eglm = __expf(gl - gm);
            float dgl = 0.f;
#pragma unroll
            for (int half = 0; half < 2; ++half) {   // 16 tokens at a time
                float dkl[16], dql[16], dkr[16];
                const uint32_t col = 32 * wg + 16 * half;
                tmem_ld16(T1 + lane_base + col, dkl);
                tmem_ld16(T1 + lane_base + 64 + col, dql);
                tmem_ld16(T2 + lane_base + col, dkr);
                tmem_wait_ld();
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const int r = (int)col + t;
                    const float gg = g[r * DK + ch];
                    const float kk = __bfloat162float(kq[r * DK + ch]), qq = __bfloat162float(kq[(kChunk + r) * DK + ch]);
                    const size_t off = (size_t)(tok0 + r) * rowk + (size_t)h * DK + ch;
                    const float d = gg - gm;
                    const float fl = __expf(d), fr = __expf(-d);
                    const float eg = egm * fl, eh = eglm * fr;   // e^{g}, e^{g_{L-1} - g}
                    const float a = dkl[t] * fl, b = dql[t] * fl, cr = dkr[t] * fr;
                    const float dkt = dktv[16 * half + t], dkh = dkhv[16 * half + t], dqt = dqtv[16 * half + t];
                    if (r < L) {
                        dk[off] = __float2bfloat16_rn(a + cr + dkt * eg + dkh * eh);
                        dq[off] = __float2bfloat16_rn(b + dqt * eg);
                    }
                    const float kh = kk * eh;
                    dgl += dkh * kh;
                    g[r * DK + ch] = kk * (a - cr + dkt * eg) - dkh * kh + qq * (b + dqt * eg);   // dg
                }
            }
            atomicAdd(&s_dgl[ch], dgl);
        }
        __syncthreads();
        // dbeta = (parts through W, U0) + rowsum(dA M)
        if (tid < L) dbeta[(size_t)(tok0 + tid) * H + h] = dbp + rowsum[tid] + rowsum[kChunk + tid];
        // dlog_alpha_s = sum_{r >= s} dg_r (+ g_{L-1}'s own cotangent), per channel
        if (gate != kGateNone && tid < DK) {
            float run = s_dgl[tid] + dgam * __expf(s_gl[tid]);
#pragma unroll 16
            for (int r = kChunk - 1; r >= 0; --r) {
                if (r < L) {
                    run += g[r * DK + tid];
                    if (gate == kGateChannel) dla[(size_t)(tok0 + r) * rowk + (size_t)h * DK + tid] = run;
                    else g[r * DK + tid] = run;
                }
            }
        }
        if (gate == kGateHead) {
            __syncthreads();
            if (tid < L) {
                float acc = 0.f;
                for (int cc = 0; cc < DK; ++cc) acc += g[tid * DK + (cc + tid) % DK];
                dla[(size_t)(tok0 + tid) * H + h] = acc;
            }
        }
        tc_fence_before();
        __syncthreads();   // g, s_beta and TMEM are free for the next item
        w = nw;
    }

    if (aborted) {
        if (tid == 0) flag_error(hdr, kStatusTimeout);
        if (mma_pending) (void)mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        if (load_pending) (void)mbar_wait_cycles(&bar_load, load_phase, kWaitCycles / 4);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// ------------------------------------------------------------- host -----
template <int DK, int DV>
cudaError_t launch_bwd_inter_tc_t(const ChunkArgs& a) {
    if (a.num_seqs == 0) return cudaSuccess;
    const int ntok = a.cu_seqlens ? a.T : a.B * a.T;
    CUtensorMap mdo;
    if (!make_map(&mdo, a.d_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DV, a.H, ntok, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    ChunkMap map{a.cu_seqlens, a.chunk_offsets, a.num_seqs, a.T, a.fixed_chunks_per_seq};
    auto kern = bwd_inter_tc_kernel<DK, DV>;
    const int smem = (int)B3Smem<DK, DV>::END + 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)a.num_seqs, (unsigned)a.H, (unsigned)(DV / kSliceTc));
    kern<<<grid, 256, smem, a.stream>>>(mdo, a.d_final_state, a.d_initial_state, a.dS_end, a.dU, map,
                                        static_cast<WsHeader*>(a.ws_header),
                                        static_cast<const unsigned char*>(a.records), a.H, a.max_chunks, a.scale);
    return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_bwd_vside_tc_t(const ChunkArgs& a) {
    if (a.max_chunks == 0) return cudaSuccess;
    const int ntok = a.cu_seqlens ? a.T : a.B * a.T;
    CUtensorMap mdo;
    if (!make_map(&mdo, a.d_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DV, a.H, ntok, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    ChunkMap map{a.cu_seqlens, a.chunk_offsets, a.num_seqs, a.T, a.fixed_chunks_per_seq};
    auto kern = bwd_vside_tc_kernel<DK, DV>;
    const int smem = (int)VsSmem<DK, DV>::END + 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const size_t items = a.max_chunks * (size_t)a.H;   // upper bound; the kernel reads the exact count
    const unsigned grid = (unsigned)(items < (size_t)sms ? items : (size_t)sms);
    kern<<<grid, 256, smem, a.stream>>>(mdo, map, static_cast<WsHeader*>(a.ws_header),
                                        static_cast<const unsigned char*>(a.records), a.states, a.dS_end, a.dU,
                                        a.vside, a.H, a.max_chunks, a.scale);
    return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_bwd_tchain_tc_t(const ChunkArgs& a) {
    if (a.max_chunks == 0) return cudaSuccess;
    ChunkMap map{a.cu_seqlens, a.chunk_offsets, a.num_seqs, a.T, a.fixed_chunks_per_seq};
    auto kern = bwd_tchain_tc_kernel<DK, DV>;
    const int smem = (int)TchSmem<DK, DV>::END + 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const size_t items = a.max_chunks * (size_t)a.H;
    const unsigned grid = (unsigned)(items < (size_t)sms ? items : (size_t)sms);
    kern<<<grid, 256, smem, a.stream>>>(map, static_cast<WsHeader*>(a.ws_header),
                                        static_cast<const unsigned char*>(a.bwd_tiles), a.dU, a.beta, a.vside,
                                        static_cast<__nv_bfloat16*>(a.dv_out), a.H, a.max_chunks);
    return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_bwd_split_tc_t(const ChunkArgs& a) {
    if (a.max_chunks == 0) return cudaSuccess;
    const int ntok = a.cu_seqlens ? a.T : a.B * a.T;
    CUtensorMap mk, mq, mla;
    if (!make_map(&mk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, a.H, ntok, DK, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&mq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, a.H, ntok, DK, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        (a.gate == kGateChannel &&
         !make_map(&mla, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, DK, a.H, ntok, DK, CU_TENSOR_MAP_SWIZZLE_NONE)))
        return cudaErrorInvalidValue;
    if (a.gate != kGateChannel) memset(&mla, 0, sizeof(mla));   // unused
    ChunkMap map{a.cu_seqlens, a.chunk_offsets, a.num_seqs, a.T, a.fixed_chunks_per_seq};
    auto kern = bwd_split_tc_kernel<DK, DV>;
    const int smem = (int)SpSmem<DK, DV>::END + 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const size_t items = a.max_chunks * (size_t)a.H;
    const unsigned grid = (unsigned)(items < (size_t)sms ? items : (size_t)sms);
    kern<<<grid, 256, smem, a.stream>>>(
        mq, mk, mla, static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k), a.log_alpha,
        a.beta, map, static_cast<WsHeader*>(a.ws_header), static_cast<const unsigned char*>(a.bwd_tiles),
        a.bwd_flags, a.vside, static_cast<__nv_bfloat16*>(a.dq), static_cast<__nv_bfloat16*>(a.dk_out),
        a.dlog_alpha, a.dbeta, a.H, a.max_chunks, a.gate);
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

size_t bwd_tiles_bytes(int dk, int dv) {
    if (dk == 128 && dv == 128) return BwdTiles<128, 128>::BYTES;
    if (dk == 128 && dv == 64) return BwdTiles<128, 64>::BYTES;
    if (dk == 64 && dv == 128) return BwdTiles<64, 128>::BYTES;
    if (dk == 64 && dv == 64) return BwdTiles<64, 64>::BYTES;
    return 0;
}

size_t tc_record_bytes(int dk, int dv) {
    if (dk == 128 && dv == 128) return TcRec<128, 128>::BYTES;
    if (dk == 128 && dv == 64) return TcRec<128, 64>::BYTES;
    if (dk == 64 && dv == 128) return TcRec<64, 128>::BYTES;
    if (dk == 64 && dv == 64) return TcRec<64, 64>::BYTES;
    return 0;
}

cudaError_t launch_chunk_intra_tc(const ChunkArgs& a) {
    // the two-CTA-per-SM kernel of kda_intra_tc.cu, which also writes the
    // backward tiles when a.bwd_tiles is set
    return launch_chunk_intra_fwd_tc(a);
}

cudaError_t launch_chunk_inter_tc(const ChunkArgs& a) {
    if (a.num_seqs == 0) return cudaSuccess;
    // the slice-width-adaptive kernel of kda_inter_tc.cu, which also writes the
    // chunk-start states when a.states is set
    return launch_chunk_inter_fwd_tc(a);
}

cudaError_t launch_chunk_bwd_inter_tc(const ChunkArgs& a) { KDA_TC_DISPATCH(launch_bwd_inter_tc_t, a); }

cudaError_t launch_chunk_bwd_vside_tc(const ChunkArgs& a) { KDA_TC_DISPATCH(launch_bwd_vside_tc_t, a); }

cudaError_t launch_chunk_bwd_tchain_tc(const ChunkArgs& a) { KDA_TC_DISPATCH(launch_bwd_tchain_tc_t, a); }

cudaError_t launch_chunk_bwd_split_tc(const ChunkArgs& a) { KDA_TC_DISPATCH(launch_bwd_split_tc_t, a); }

}  // namespace kda
