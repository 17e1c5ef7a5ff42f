// kda_intra_tc.cu -- the forward intra-chunk kernel on the sm_100a tensor cores
// (bf16 inputs), two CTAs per SM.
//
// Per (chunk, head) item, with g_r = sum_{i<=r} log alpha_i per key channel
// and g_m the middle token's (the chunk algebra of the chunk-wise parallel
// form, kongchang.com "Kimi Delta Attention详解", section "硬件效率的优化策略",
// obtained by unrolling the daiw.net update equation, section "KDA 的更新式"):
//
//   [A; P] = [K~m; Q~m] K-m^T  (tf32, A operand in TMEM, B in shared memory)
//   T = (I + A)^{-1}: 16 x 16 diagonal blocks on CUDA cores (fp32), the rest by
//       blocked doubling on the tensor cores (fp16 operands)
//   W = T diag(beta) K~,  U0 = T diag(beta) V  (fp16 operands)
//   records: W, Q~ = q e^{g}, K^ = k e^{g_{L-1} - g}, P, U0 (fp16), gamma_C (fp32)
//
// The records have the layout the inter-chunk kernel reads (TcRec).  In
// backward mode (a separate instance) the kernel also writes what the backward
// kernels read (BwdTiles: fp16 T, K~ and V tiles, the fp32 M = K_l K_r^T, a
// strong-decay flag).  MMA1's 128-row A operand stays in tensor memory instead
// of 64 KB of shared memory, the log-decay tile comes in a 128-byte-swizzled
// layout that both the per-channel scan and the per-row element pass read
// without bank conflicts, and v is loaded only after the element pass.  That
// brings a CTA to about 108 KB of shared memory, 256 TMEM columns
// and at most 128 registers per thread, so two CTAs share each SM and one item's
// latency-bound phases (the (I + A)^{-1} solve, the TMEM round trips, the
// copies) overlap the other CTA's work.
//
// Each wait on an mbarrier is done by one thread (bounded); the others block at
// the CTA barrier that follows, so a waiting CTA issues no instructions and
// leaves the SM's issue slots to the other CTA.  The waiting thread's acquire
// of the phase and the barrier order the copies / MMAs before every thread's
// later accesses.  A CTA that gives up records KDA_ERR_TIMEOUT, drains exactly
// the copies and MMAs it issued, frees its tensor memory and returns.
#include <cuda_fp16.h>

#include <cstring>
#include <type_traits>

#include "kda_common.cuh"
#include "kda_launch.h"
#include "kda_tc_common.cuh"
#include "ptx.cuh"

namespace kda {
namespace {

using namespace ptx;

// Shared memory of one CTA (byte offsets; tiles of 64 rows x 128 bytes, 128-byte swizzled).
template <int DK, int DV, bool FUSED>
struct K1fSmem {
    static constexpr uint32_t TILE = 8192;
    // T diag(beta), rows 0..63: MMA2's 128-row A operand, whose unused rows
    // 64..127 are the first 8 KB of KT right behind it
    static constexpr uint32_t TPV = 0;
    static constexpr uint32_t KT = TPV + TILE;                          // k (bf16) -> K~ (fp16, MMA2 B)
    static constexpr uint32_t KT_BYTES = (DK / 64) * TILE;
    static constexpr uint32_t QT = KT + KT_BYTES;                       // q -> Q~ (fp16); the next item's q
    static constexpr uint32_t QT_BYTES = (DK / 64) * TILE;
    static constexpr uint32_t G = QT + QT_BYTES;                        // log_alpha -> g (fp32, 32-channel tiles)
    static constexpr uint32_t G_BYTES = 64 * DK * 4;
    static constexpr uint32_t VT = G;                                   // after the element pass: v -> V (MMA2 B)
    static constexpr uint32_t VB = (DV / 64) * TILE;
    static constexpr uint32_t OPB = G + G_BYTES;                        // K-m tf32 (MMA1 B); W | U0 fp16 staging
    static constexpr uint32_t OPB_BYTES = (DK / 32) * TILE;
    static constexpr uint32_t STG_BYTES = ((DK + DV) / 64) * TILE;
    // after MMA1, behind V: fp32 scratch of the first (CUDA-core) level of the
    // blocked (I + A)^{-1} (A's blocks (1,0) and (3,2), their products, the
    // diagonal inverses D), then the fp16 operands of its tensor-core level (A
    // masked to its lower-left quadrant, a product X, T restricted to its 32 x 32
    // diagonal blocks), each 64 x 64 tile read as a 128-row operand whose rows
    // 64..127 are the next 8 KB; then A's four diagonal 16 x 16 blocks in fp32
    // (padded).  The strong-decay path writes the full fp32 A ([64][64]) before
    // the element pass, while g is live, outside G and clear of AF, AH2 and AMD.
    static constexpr uint32_t SCR = G + VB;
    static constexpr uint32_t AF = SCR;                                 // [2][16][17] fp32 A_10, A_32
    static constexpr uint32_t XF = SCR + 2304;                          // [2][16][17] fp32 A_10 D_0, A_32 D_2
    static constexpr uint32_t AH2 = SCR + 8192;
    static constexpr uint32_t DF = SCR + 16384;                         // [4][16][17] fp32 D_0..D_3
    static constexpr uint32_t XH = SCR + 24576;
    static constexpr uint32_t T1H = SCR + 32768;
    static constexpr uint32_t AMD = SCR + 40960;                        // 4 x (16 x 16 + 4) fp32
    static constexpr uint32_t AMD_END = AMD + 4 * 260 * 4;
    static constexpr uint32_t AMS0 = (G + G_BYTES) > (AH2 + 8192) ? (G + G_BYTES) : (AH2 + 8192);
    static constexpr uint32_t AMS = AMS0 + 64 * 64 * 4 <= AMD ? AMS0 : (AMD_END + 15) / 16 * 16;   // [64][64]
    // log-decay boxes (32 channels, 8 KB) past V overlap only AF, XF, AH2 and DF,
    // which are dead once the second blocked-inverse level has read AH2: the
    // next item's boxes there are fetched then, the others after MMA2
    static constexpr int LA_EARLY_BOX = (int)(VB / TILE);
    static constexpr uint32_t E0 = OPB + (OPB_BYTES > STG_BYTES ? OPB_BYTES : STG_BYTES);
    static constexpr uint32_t E1 = T1H + 16384;                          // T1H's rows 64..127 end here
    static constexpr uint32_t E2 = AMS + 64 * 64 * 4;
    static constexpr uint32_t E3 = AMD_END;
    static constexpr uint32_t E01 = E0 > E1 ? E0 : E1;
    static constexpr uint32_t E23 = E2 > E3 ? E2 : E3;
    static constexpr uint32_t END0 = ((E01 > E23 ? E01 : E23) + 1023) / 1024 * 1024;
    // fused form only: the chunk's operands of the state step, kept on chip ---
    // [W; Q~] as 128-row K-major tiles per 64 key channels, K^ and P (P
    // directly after K^, so the 128-row operand [*; P] reads K^'s tail as its
    // unused rows 0..63), gamma_C, the fp16 state (rows = key channel) and U
    // operands of the state step; U0 where K-m was
    static constexpr int NTV = DV > 64 ? DV / 64 : 1;
    static constexpr uint32_t FWQ = END0;
    static constexpr uint32_t FU0 = OPB;   // written after MMA2, when OPB (K-m, the solve's scratch) is dead
    static constexpr uint32_t FKH = FWQ + (DK / 64) * 16384;
    static constexpr uint32_t FP = FKH + (DK / 64) * TILE;
    static constexpr uint32_t S16 = FP + TILE;
    static constexpr uint32_t U16 = S16 + NTV * 16384;
    static constexpr uint32_t FGC = U16 + NTV * TILE;
    static constexpr uint32_t END = FUSED ? FGC + DK * 4 : END0;
    static constexpr uint32_t BAR = END;                                 // bar_in, bar_v, bar_mma
    static constexpr uint32_t TMEMADDR = BAR + 24;
    static constexpr uint32_t BETA = BAR + 32;                           // [64]
    static constexpr uint32_t GM = BETA + 256;                           // [DK] g_m (base 2)
    static constexpr uint32_t EGM = GM + DK * 4;                         // [DK] e^{g_m}
    static constexpr uint32_t EGLM = EGM + DK * 4;                       // [DK] e^{g_{L-1} - g_m}
    static constexpr uint32_t LAH = EGLM + DK * 4;                       // [64] per-head log-decay
    static constexpr uint32_t PART = LAH + 256;                          // [256 / DK][DK] scan partials
    static constexpr uint32_t PAIR = PART + 256 * 4;                     // fused: the claimed pair
    static constexpr uint32_t TOTAL = PAIR + 16;
    static constexpr uint32_t KQ_TX = 2 * (DK / 64) * TILE;              // k and q tiles
    static constexpr uint32_t LA_TX = 64 * DK * 4;
    static constexpr uint32_t V_TX = (DV / 64) * TILE;
    static_assert(KT == TPV + 8192 && TPV % 1024 == 0 && OPB % 1024 == 0 && G % 1024 == 0 && SCR % 1024 == 0,
                  "swizzled tiles need 1024-byte alignment; MMA2's A operand runs into KT");
    static_assert(AMS >= G + G_BYTES && AMS >= AH2 + 8192 && (AMS + 64 * 64 * 4 <= AMD || AMS >= AMD_END),
                  "the strong path's A lies outside the live log-decay tile and the converted operands");
    static_assert(XF + 2 * 16 * 17 * 4 <= AH2 && DF + 4 * 16 * 17 * 4 <= XH, "level-1 scratch");
    static_assert(G + G_BYTES <= SCR + 24576, "early log-decay boxes overlap only AF, XF, AH2, DF");
    // two CTAs per SM (228 KB per SM, 1 KB reserved per CTA); the fused form one
    static_assert(FUSED ? TOTAL <= 232448 : 2 * (TOTAL + 1024) <= 233472, "CTAs per SM");
    static_assert(FWQ % 1024 == 0 && S16 % 1024 == 0, "swizzled tiles need 1024-byte alignment");
    static_assert((DV / 64) * TILE <= OPB_BYTES, "the fused U0 fits where K-m was");
};

// g (base 2) of token r, channel c in the 128-byte-swizzled log-decay tiles
// (32 channels x 64 tokens each).
__device__ __forceinline__ uint32_t g_off(int r, int c) {
    return (uint32_t)(c >> 5) * 8192u + sw128_offset((uint32_t)r, (uint32_t)(c & 31) * 4u);
}

template <int DK, int DV, int GATE, bool FUSED, bool BWD>
__global__ void __launch_bounds__(256, FUSED ? 1 : 2)
intra_chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_la,
                          const float* __restrict__ log_alpha_head, const float* __restrict__ beta,
                          ChunkMap map, WsHeader* hdr, unsigned char* __restrict__ records, int H,
                          size_t max_chunks, long long wait_cap, int drop_la,
                          const float* __restrict__ initial_state, float* __restrict__ final_state,
                          __nv_bfloat16* __restrict__ o, float scale, const int* __restrict__ seq_order,
                          unsigned char* __restrict__ bwd_tiles, int* __restrict__ bwd_flags)
{
    using Sm = K1fSmem<DK, DV, FUSED>;
    using R = TcRec<DK, DV>;
    using BT = BwdTiles<DK, DV>;
    constexpr int NPART = 256 / DK;       // threads per key channel in the scan
    constexpr int TPP = kChunk / NPART;   // tokens per such thread
    constexpr int CH = DK / 2;            // channels per thread in the element pass
    constexpr bool channel_gate = GATE == kGateChannel;
    extern __shared__ __align__(1024) unsigned char sm[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Sm::BAR);
    uint64_t& bar_in = bars[0];    // k, q (and log_alpha) of an item
    uint64_t& bar_v = bars[1];     // v of an item
    uint64_t& bar_mma = bars[2];
    uint32_t& s_tmem = *reinterpret_cast<uint32_t*>(sm + Sm::TMEMADDR);
    float* s_beta = reinterpret_cast<float*>(sm + Sm::BETA);
    float* s_gm = reinterpret_cast<float*>(sm + Sm::GM);
    float* s_egm = reinterpret_cast<float*>(sm + Sm::EGM);
    float* s_eglm = reinterpret_cast<float*>(sm + Sm::EGLM);
    float* s_lah = reinterpret_cast<float*>(sm + Sm::LAH);
    float* s_part = reinterpret_cast<float*>(sm + Sm::PART);

    if (hdr->status != kStatusOk) return;
    const int total = hdr->num_chunks * H;
    if (!FUSED && (int)blockIdx.x >= total) return;
    if ((smem_u32(sm) & 1023u) != 0) {   // the swizzled layouts need 1024-byte alignment
        if (threadIdx.x == 0) flag_error(hdr, kStatusInternal);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ch = tid % DK, part = tid / DK, r0 = part * TPP;   // scan mapping
    const int row = 32 * (warp & 3) + lane;                      // TMEM lane: 0..63 K rows, 64..127 Q rows
    const int hc = warp >> 2;                                    // channel half of the element pass
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;

    if (tid == 0) {
        mbar_init(&bar_in, 1);
        mbar_init(&bar_v, 1);
        mbar_init(&bar_mma, 1);
        fence_mbar_init();
    }
    constexpr uint32_t kTmemCols = FUSED ? 512 : 256;
    if (warp == 0) {
        tmem_alloc(&s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const uint32_t AOP = tmem;        // [K~m; Q~m] tf32, 128 lanes x DK columns
    const uint32_t D1 = tmem + DK;    // [A; P], 128 lanes x 64 columns
    const uint32_t D2 = tmem;         // [W | U0], lanes 0..63 x (DK + DV) columns (after D1 is read)
    const uint32_t R3 = tmem;         // fused: [W S; Q~ S + P U], 128 lanes x DV (after D2 is read)
    const uint32_t SACC = tmem + kTmemCols - DV;   // fused: the fp32 state, lanes 0..DK-1 x DV

    // test hook: CTA 0 can leave out the log-decay copy of its third item (of
    // its last if it has fewer), so that the bounded wait on that item's
    // inputs gives up with earlier phases consumed
    const int drop_it = (!FUSED && drop_la && blockIdx.x == 0) ? min(2, (total - 1) / (int)gridDim.x) : -1;
    // An item's inputs arrive in three parts as their buffers free up: q (QT is
    // free once the previous item's Q~ has left it), the log-decay boxes past V
    // (free after the second blocked-inverse level), then k and the other boxes
    // (after MMA2).  All land on bar_in, armed with the whole byte count by the
    // first part.  (h, tok0): the item's head and first token; j: this CTA's
    // item count at that item.
    auto issue_q = [&](int h, int tok0) {
        mbar_arrive_expect_tx(&bar_in, Sm::KQ_TX + (channel_gate ? Sm::LA_TX : 0u));
#pragma unroll
        for (int b = 0; b < DK / 64; ++b) tma_load_3d(sm + Sm::QT + b * Sm::TILE, &tm_q, &bar_in, b * 64, h, tok0);
    };
    auto issue_la = [&](int h, int tok0, int j, bool early) {
        if constexpr (channel_gate) {
            if (j == drop_it) return;   // test hook: this item's log-decay copy is left out
#pragma unroll
            for (int b = 0; b < DK / 32; ++b)
                if ((b >= Sm::LA_EARLY_BOX) == early)
                    tma_load_3d(sm + Sm::G + b * Sm::TILE, &tm_la, &bar_in, b * 32, h, tok0);
        }
    };
    auto issue_k = [&](int h, int tok0) {
#pragma unroll
        for (int b = 0; b < DK / 64; ++b) tma_load_3d(sm + Sm::KT + b * Sm::TILE, &tm_k, &bar_in, b * 64, h, tok0);
    };
    auto issue_in = [&](int c, int h, int j) {   // all of chunk c, head h at once
        int seq, tok0, L;
        map.locate(c, seq, tok0, L);
        issue_q(h, tok0);
        issue_la(h, tok0, j, true);
        issue_la(h, tok0, j, false);
        issue_k(h, tok0);
    };
    // beta (and a per-head log-decay) of item w into registers, threads 192..255
    float beta_next = 0.f, lah_next = 0.f;
    auto load_beta = [&](int c, int h) {
        if (tid >= 192) {
            int seq, tok0, L;
            map.locate(c, seq, tok0, L);
            const int r = tid - 192;
            beta_next = (r < L) ? ld_prefetch_f32(beta + (size_t)(tok0 + r) * H + h) : 0.f;
            lah_next = (GATE == kGateHead && r < L) ? ld_prefetch_f32(log_alpha_head + (size_t)(tok0 + r) * H + h) : 0.f;
        }
    };

    bool aborted = false;
    uint32_t mma_phase = 0;
    int mma_pending = 0;          // a commit on bar_mma not yet waited for
    // this CTA's j-th item lands on bar_in / bar_v with phase parity j & 1;
    // items [in_done, in_issued) and [v_done, v_issued) are in flight
    int in_issued = 0, in_done = 0, v_issued = 0, v_done = 0;
    bool stored = false;          // the copy thread has bulk stores in flight
    float range_max = 0.f;

    int it = 0;   // this CTA's item count
    // One (chunk c, head h) item of L tokens from token tok0; (nc, nh) is this
    // CTA's next item (nc < 0: none), prefetched once this one's inputs are
    // consumed.  Returns false if a wait gave up.
    auto run_item = [&](int c, int h, int tok0, int L, int nc, int nh) -> bool {
        unsigned char* rec = records + ((size_t)h * max_chunks + c) * R::BYTES;
        // where the chunk's intermediates go: the record (split form) or the
        // on-chip operands of the state step (fused form)
        float* gc_dst = FUSED ? reinterpret_cast<float*>(sm + Sm::FGC) : reinterpret_cast<float*>(rec + R::GC);
        unsigned char* kh_dst = FUSED ? sm + Sm::FKH : rec + R::KH;
        unsigned char* p_dst = FUSED ? sm + Sm::FP : rec + R::P;
        // backward mode (split form): T = (I + A)^{-1}, K~ and V as fp16 tiles and the
        // unweighted M = K_l K_r^T for the backward's T-chain and split-factor kernels
        unsigned char* btile = (BWD && !FUSED) ? bwd_tiles + ((size_t)h * max_chunks + c) * BT::BYTES : nullptr;
        if (tid >= 192) {
            s_beta[tid - 192] = beta_next;
            if constexpr (GATE == kGateHead) s_lah[tid - 192] = lah_next;
        }
        if (nc >= 0) load_beta(nc, nh);
        int ntok0 = 0;   // the next item's first token (copy thread)
        if (tid == kCopyThread && nc >= 0) {
            int sq, nl;
            map.locate(nc, sq, ntok0, nl);
        }
        // the previous item's W / U0 staging (OPB) must be read before it is reused
        if (tid == kCopyThread && stored) bulk_store_wait_read();

        // ---- cumulative log-decay, in place over the log_alpha tile in G -------
        const bool ok_in = (!FUSED && tid != 0) || mbar_wait_cycles(&bar_in, it & 1, wait_cap);
        if (__syncthreads_or(!ok_in)) return false;
        in_done = it + 1;
        {
            float la_cur[TPP];
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < TPP; ++i) {
                if constexpr (channel_gate) la_cur[i] = (r0 + i < L) ? *reinterpret_cast<const float*>(sm + Sm::G + g_off(r0 + i, ch)) : 0.f;
                else if constexpr (GATE == kGateHead) la_cur[i] = (r0 + i < L) ? s_lah[r0 + i] : 0.f;
                else la_cur[i] = 0.f;   // no gate: alpha = 1
                acc += la_cur[i];
            }
            s_part[part * DK + ch] = acc;
            __syncthreads();
            acc = 0.f;
            for (int p = 0; p < part; ++p) acc += s_part[p * DK + ch];
#pragma unroll
            for (int i = 0; i < TPP; ++i) {
                acc += la_cur[i];
                *reinterpret_cast<float*>(sm + Sm::G + g_off(r0 + i, ch)) = acc * kLog2e;   // base 2
            }
        }
        __syncthreads();
        auto gat = [&](int r, int cc) { return *reinterpret_cast<const float*>(sm + Sm::G + g_off(r, cc)); };
        bool wide = false;   // this channel's decay within the chunk too strong for the split factors
        if (tid < DK) {
            const float gm = gat((L - 1) >> 1, tid), gl = gat(L - 1, tid);   // base 2
            s_gm[tid] = gm;
            s_egm[tid] = ex2_approx(gm);
            s_eglm[tid] = ex2_approx(gl - gm);
            gc_dst[tid] = exp2f(gl);
            wide = fmaxf(gat(0, tid) - gm, gm - gl) > kMaxSplitExponent2;
        }
        // Strong decay: the factors e^{+-(g - g_m)} of A and P could overflow, so
        // this chunk forms A and P exactly (slow path, no MMA1).
        const bool strong = __syncthreads_or(wide);
        if (BWD && !FUSED && tid == 0) bwd_flags[(size_t)h * max_chunks + c] = strong ? 1 : 0;
        float* am = reinterpret_cast<float*>(sm + Sm::AMS);   // strong path: [64][64]
        if (strong) {
            exact_a_p<DK>(gat, sm + Sm::KT, sm + Sm::QT, s_beta, L, am, p_dst, 64);
            __syncthreads();   // the k, q tiles are converted in place next
        }

        // ---- element pass: thread -> TMEM lane `row`, channels [CH hc, CH hc + CH).
        //      K rows (0..63, token r) form everything that comes from k: K~m ->
        //      TMEM and K-m -> OPB (tf32), K~ = k e^{g} -> KT in place (fp16),
        //      K^ = k e^{g_{L-1} - g} -> record (fp16).  Q rows (64..127) form
        //      Q~m -> TMEM (tf32) and Q~ = q e^{g} -> QT in place (fp16).  Each
        //      thread overwrites only the tile row it read.
        const bool is_k = row < 64;
        const int er = row & 63;
        const bool live = er < L;
        auto element_pass = [&](auto strong_tag) {
            constexpr bool STRONG = decltype(strong_tag)::value;
#pragma unroll 2
            for (int j = 0; j < CH / 8; ++j) {
                const int c8 = CH * hc + 8 * j;
                const uint32_t ho = (uint32_t)(c8 >> 6) * Sm::TILE + sw128_offset(er, (c8 & 63) * 2);
                unsigned char* xt = sm + (is_k ? Sm::KT : Sm::QT) + ho;   // this row's k or q chunk
                // K~ goes back in place (MMA2's operand); Q~ in place (split form:
                // bulk-stored to the record) or into the fused [W; Q~] operand
                unsigned char* xo = (FUSED && !is_k)
                    ? sm + Sm::FWQ + (uint32_t)(c8 >> 6) * 16384 + 8192 + sw128_offset(er, (c8 & 63) * 2) : xt;
                uint4 raw = *reinterpret_cast<const uint4*>(xt);
                if (!live) raw = make_uint4(0, 0, 0, 0);
                const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(&raw);
                const float4 g0 = *reinterpret_cast<const float4*>(sm + Sm::G + g_off(er, c8));
                const float4 g1 = *reinterpret_cast<const float4*>(sm + Sm::G + g_off(er, c8 + 4));
                const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                uint32_t top[8];                      // tf32 bits of K~m / Q~m (TMEM)
                __align__(16) float kbm[8];           // K-m (OPB)
                __align__(16) __half2 h0[4], h1[4];   // K~ | Q~ (in place), K^ (record)
                if constexpr (!STRONG) {
                    const float4 m0 = *reinterpret_cast<const float4*>(s_gm + c8);
                    const float4 m1 = *reinterpret_cast<const float4*>(s_gm + c8 + 4);
                    const float4 x0 = *reinterpret_cast<const float4*>(s_egm + c8);
                    const float4 x1 = *reinterpret_cast<const float4*>(s_egm + c8 + 4);
                    const float gmv[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
                    const float egmv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    if (is_k) {
                        const float4 y0 = *reinterpret_cast<const float4*>(s_eglm + c8);
                        const float4 y1 = *reinterpret_cast<const float4*>(s_eglm + c8 + 4);
                        const float eglmv[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            float t[2], u2[2];
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const int e = 2 * e2 + u;
                                const float kk = __bfloat162float(xb[e]);
                                const float d = gv[e] - gmv[e];
                                const float kem = kk * ex2_approx(d);           // k e^{g_r - g_m}
                                const float keb = kk * ex2_approx(-d);          // k e^{g_m - g_r}
                                top[e] = __float_as_uint(round_tf32_alu(kem));
                                kbm[e] = round_tf32_alu(keb);
                                t[u] = kem * egmv[e];                           // k e^{g_r}
                                u2[u] = keb * eglmv[e];                         // k e^{g_{L-1} - g_r}
                            }
                            h0[e2] = __floats2half2_rn(t[0], t[1]);
                            h1[e2] = __floats2half2_rn(u2[0], u2[1]);
                        }
                        const uint32_t fo = (uint32_t)(c8 >> 5) * Sm::TILE, fb = (c8 & 31) * 4;
                        *reinterpret_cast<float4*>(sm + Sm::OPB + fo + sw128_offset(er, fb)) = *reinterpret_cast<const float4*>(kbm);
                        *reinterpret_cast<float4*>(sm + Sm::OPB + fo + sw128_offset(er, fb + 16)) = *reinterpret_cast<const float4*>(kbm + 4);
                        *reinterpret_cast<uint4*>(kh_dst + ho) = *reinterpret_cast<const uint4*>(h1);
                    } else {
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            float t[2];
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const int e = 2 * e2 + u;
                                const float qem = __bfloat162float(xb[e]) * ex2_approx(gv[e] - gmv[e]);   // q e^{g_r - g_m}
                                top[e] = __float_as_uint(round_tf32_alu(qem));
                                t[u] = qem * egmv[e];                                                   // q e^{g_r}
                            }
                            h0[e2] = __floats2half2_rn(t[0], t[1]);
                        }
                    }
                    *reinterpret_cast<uint4*>(xo) = *reinterpret_cast<const uint4*>(h0);
                    tmem_st8(AOP + lane_base + c8, top);
                } else {   // strong-decay chunk: unsplit factors, every exponent <= 0; no MMA1 operands
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        float t[2], u2[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int e = 2 * e2 + u;
                            const float x = __bfloat162float(xb[e]);
                            t[u] = x * ex2_approx(gv[e]);                                          // k e^{g_r} | q e^{g_r}
                            u2[u] = is_k ? x * ex2_approx(gat(L - 1, c8 + e) - gv[e]) : 0.f;       // k e^{g_{L-1} - g_r}
                        }
                        h0[e2] = __floats2half2_rn(t[0], t[1]);
                        h1[e2] = __floats2half2_rn(u2[0], u2[1]);
                    }
                    *reinterpret_cast<uint4*>(xo) = *reinterpret_cast<const uint4*>(h0);
                    if (is_k) *reinterpret_cast<uint4*>(kh_dst + ho) = *reinterpret_cast<const uint4*>(h1);
                }
            }
        };
        if (strong) element_pass(std::true_type{});
        else element_pass(std::false_type{});
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && !strong) {
            // ---- MMA1 (tf32, A from TMEM): [K~m; Q~m] K-m^T -> D1
            tc_fence_after();
            constexpr uint32_t idesc = instr_desc(kFmtTF32, 128, 64);
            const uint32_t b0 = smem_u32(sm + Sm::OPB);
#pragma unroll
            for (int kb = 0; kb < DK / 32; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_tf32_ts(D1, AOP + kb * 32 + ks * 8, smem_desc(b0 + kb * 8192 + ks * 32, 16, 1024, kLayoutSW128),
                                idesc, (kb | ks) != 0);
            mma_commit(&bar_mma);
        }
        mma_pending = strong ? 0 : 1;
        if (tid == kCopyThread) {
            if constexpr (!FUSED) {
                // Q~ tiles are the lower halves (rows 64..127) of the record's WQ
                // tiles; once they are read, v comes into the same buffer
#pragma unroll
                for (int b = 0; b < DK / 64; ++b)
                    bulk_store(rec + R::WQ + b * 16384 + 8192, sm + Sm::QT + b * Sm::TILE, 8192);
                if (btile)   // backward mode: K~ is final in KT
                    bulk_store(btile + BT::KT, sm + Sm::KT, (DK / 64) * Sm::TILE);
                bulk_store_commit();
                stored = true;
                bulk_store_wait_read();
            }
            // v into the log-decay tile's place (g is dead after the element pass)
            mbar_arrive_expect_tx(&bar_v, Sm::V_TX);
#pragma unroll
            for (int b = 0; b < DV / 64; ++b) tma_load_3d(sm + Sm::VT + b * Sm::TILE, &tm_v, &bar_v, b * 64, h, tok0);
            if (nc >= 0) issue_q(nh, ntok0);   // QT is free: the next item's q
        }
        v_issued = it + 1;
        if (nc >= 0) in_issued = it + 2;

        float* amd = reinterpret_cast<float*>(sm + Sm::AMD);  // A's diagonal blocks, [4][16 x 16 + 4]
        // A row `row` (< 64), columns [32 hc, 32 hc + 32), beta-scaled and strictly
        // lower: its diagonal block -> AMD and blocks (1,0), (3,2) -> AF (fp32);
        // rows 32..63 x columns 0..31 -> AH2 (fp16, zero elsewhere)
        auto put_a_row = [&](const float (&v)[32]) {
            const int b = row >> 4;
            if ((b >> 1) == hc) {   // the diagonal block is columns [0, 16) or [16, 32) of v
                float* dst = amd + b * 260 + (row & 15) * 16;
                if ((b & 1) == 0) {
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)
                        *reinterpret_cast<float4*>(dst + 4 * k4) = make_float4(v[4 * k4], v[4 * k4 + 1], v[4 * k4 + 2], v[4 * k4 + 3]);
                } else {
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)
                        *reinterpret_cast<float4*>(dst + 4 * k4) =
                            make_float4(v[16 + 4 * k4], v[16 + 4 * k4 + 1], v[16 + 4 * k4 + 2], v[16 + 4 * k4 + 3]);
                }
            }
#pragma unroll
            for (int i8 = 0; i8 < 4; ++i8) {
                const int col = 32 * hc + 8 * i8, cb = col >> 4;
                const bool l1 = (b == 1 && cb == 0) || (b == 3 && cb == 2);
                const bool l2 = b >= 2 && cb < 2;
                __align__(16) __half h2[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) h2[e] = __float2half_rn(l2 ? v[8 * i8 + e] : 0.f);
                *reinterpret_cast<uint4*>(sm + Sm::AH2 + sw128_offset(row, col * 2)) = *reinterpret_cast<const uint4*>(h2);
                if (l1) {
                    float* af = reinterpret_cast<float*>(sm + Sm::AF) + (b >> 1) * 272 + (row & 15) * 17 + (col & 15);
#pragma unroll
                    for (int e = 0; e < 8; ++e) af[e] = v[8 * i8 + e];
                }
            }
        };
        bool ok = true;
        if (!strong) {
            ok = (!FUSED && tid != 0) || mbar_wait_cycles(&bar_mma, mma_phase, wait_cap);
            if (__syncthreads_or(!ok)) return false;
            mma_phase ^= 1;
            mma_pending = 0;
            tc_fence_after();
            // ---- A (rows 0..63) to the T-solve operands; P (rows 64..127, lower
            //      incl. diagonal) to the record
            float v[32];
            tmem_ld32_sync(D1 + lane_base + 32 * hc, v);
            if (row < 64) {
                if (btile) {   // backward mode: the unweighted, strictly lower M
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const int col = 32 * hc + 4 * i4;
                        *reinterpret_cast<float4*>(btile + BT::M + (row * 64 + col) * 4) =
                            make_float4(col < row ? v[4 * i4] : 0.f, col + 1 < row ? v[4 * i4 + 1] : 0.f,
                                        col + 2 < row ? v[4 * i4 + 2] : 0.f, col + 3 < row ? v[4 * i4 + 3] : 0.f);
                    }
                }
                const float b = s_beta[row];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = (32 * hc + i < row) ? b * v[i] : 0.f;
                put_a_row(v);
            } else {
                const int r = row - 64;
#pragma unroll
                for (int i8 = 0; i8 < 4; ++i8) {
                    __align__(16) __half hv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int col = 32 * hc + 8 * i8 + e;
                        hv[e] = __float2half_rn(col <= r ? v[8 * i8 + e] : 0.f);
                    }
                    *reinterpret_cast<uint4*>(p_dst + sw128_offset(r, (32 * hc + 8 * i8) * 2)) =
                        *reinterpret_cast<const uint4*>(hv);
                }
            }
        } else if (row < 64) {   // strong decay: the exact A, already beta-scaled and masked
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = am[row * 64 + 32 * hc + i];
            put_a_row(v);
        }
        __syncthreads();

        // ---- T = (I + A)^{-1}: exact inverses D_b = (I + A_bb)^{-1} of the four
        //      diagonal 16 x 16 blocks on CUDA cores, then the off-diagonal blocks by
        //      doubling the solved block, T21 = -T22 A21 T11: for 16 -> 32 rows (the
        //      pairs (1,0), (3,2)) on CUDA cores in fp32, for 32 -> 64 on the tensor
        //      cores (fp16 operands, fp32 accumulation).  T diag(beta) goes to TPV in
        //      fp16 (K-major, rows 0..63) block by block.
        auto put_t = [&](int rr, int col, float t) {
            *reinterpret_cast<__half*>(sm + Sm::TPV + sw128_offset(rr, col * 2)) = __float2half_rn(t * s_beta[col]);
        };
        if (tid < 64) {    // diagonal blocks, one column per thread
            const int b = tid >> 4, cc = tid & 15, base = 16 * b;
            float x[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float* arow = amd + b * 260 + j * 16;
                float av[16];
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    const float4 t4 = *reinterpret_cast<const float4*>(arow + 4 * k4);
                    av[4 * k4] = t4.x; av[4 * k4 + 1] = t4.y; av[4 * k4 + 2] = t4.z; av[4 * k4 + 3] = t4.w;
                }
                float acc4[4] = {(j == cc) ? 1.f : 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int k = 0; k < j; ++k) acc4[k & 3] -= av[k] * x[k];
                x[j] = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
                reinterpret_cast<float*>(sm + Sm::DF)[b * 272 + j * 17 + cc] = x[j];
                *reinterpret_cast<__half*>(sm + Sm::T1H + sw128_offset(base + j, (base + cc) * 2)) = __float2half_rn(x[j]);
                put_t(base + j, base + cc, x[j]);
                if (btile) *reinterpret_cast<__half*>(btile + BT::T + sw128_offset(base + j, (base + cc) * 2)) = __float2half_rn(x[j]);
            }
        } else {           // zero chunks: T1 off its diagonal and level-1 blocks, T diag(beta) above the diagonal
            for (int o = tid - 64; o < 64 * 8; o += 192) {
                const int rr = o >> 3, c16 = o & 7, blk = c16 >> 1, rb = rr >> 4;
                const bool l1 = (rb == 1 && blk == 0) || (rb == 3 && blk == 2);
                if (blk != rb && !l1) *reinterpret_cast<uint4*>(sm + Sm::T1H + sw128_offset(rr, c16 * 16)) = make_uint4(0u, 0u, 0u, 0u);
                if (blk > rb) {
                    *reinterpret_cast<uint4*>(sm + Sm::TPV + sw128_offset(rr, c16 * 16)) = make_uint4(0u, 0u, 0u, 0u);
                    if (btile) *reinterpret_cast<uint4*>(btile + BT::T + sw128_offset(rr, c16 * 16)) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
        }
        // one 64 x 64 x 64 product D[0, 64) = A(128-row K-major operand) B(64 x 64, rows = K)
        auto level_mma = [&](uint32_t a_off, uint32_t b_off) -> bool {
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                constexpr uint32_t idl = instr_desc(kFmtF16, 128, 64, false, true);
                const uint32_t a0 = smem_u32(sm + a_off), b0 = smem_u32(sm + b_off);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(tmem, smem_desc(a0 + ks * 32, 16, 1024, kLayoutSW128),
                            smem_desc(b0 + ks * 2048, Sm::TILE, 1024, kLayoutSW128), idl, ks != 0);
                mma_commit(&bar_mma);
            }
            mma_pending = 1;
            const bool good = (!FUSED && tid != 0) || mbar_wait_cycles(&bar_mma, mma_phase, wait_cap);
            if (__syncthreads_or(!good)) return false;
            mma_phase ^= 1;
            mma_pending = 0;
            tc_fence_after();
            return true;
        };
        // rows 0..63 of the product (warps 0, 1, 4, 5), as fp16 into a 64 x 64 tile
        auto store_x = [&](uint32_t dst) {
            if (row < 64) {
                float v[32];
                tmem_ld32_sync(tmem + lane_base + 32 * hc, v);
#pragma unroll
                for (int i8 = 0; i8 < 4; ++i8) {
                    __align__(16) __half hv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) hv[e] = __float2half_rn(v[8 * i8 + e]);
                    *reinterpret_cast<uint4*>(sm + dst + sw128_offset(row, (32 * hc + 8 * i8) * 2)) = *reinterpret_cast<const uint4*>(hv);
                }
            }
        };
        // level 1 (CUDA cores, fp32): X_p = A_{2p+1,2p} D_{2p}, T_{2p+1,2p} = -D_{2p+1} X_p
        //      for p = 0, 1; two entries of one row per thread
        __syncthreads();   // D and A's level-1 blocks are complete
        {
            const int pp = tid >> 7, i = (tid & 127) >> 3, j0 = (tid & 7) * 2;
            const float* af = reinterpret_cast<const float*>(sm + Sm::AF) + pp * 272 + i * 17;
            const float* d0 = reinterpret_cast<const float*>(sm + Sm::DF) + (2 * pp) * 272 + j0;
            float x0 = 0.f, x1 = 0.f;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                x0 = fmaf(af[m], d0[m * 17], x0);
                x1 = fmaf(af[m], d0[m * 17 + 1], x1);
            }
            float* xf = reinterpret_cast<float*>(sm + Sm::XF) + pp * 272 + i * 17 + j0;
            xf[0] = x0;
            xf[1] = x1;
            __syncthreads();
            const float* d1 = reinterpret_cast<const float*>(sm + Sm::DF) + (2 * pp + 1) * 272 + i * 17;
            const float* xc = reinterpret_cast<const float*>(sm + Sm::XF) + pp * 272 + j0;
            float t0 = 0.f, t1 = 0.f;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                t0 = fmaf(d1[m], xc[m * 17], t0);
                t1 = fmaf(d1[m], xc[m * 17 + 1], t1);
            }
            const int rr = 16 * (2 * pp + 1) + i, cc = 16 * (2 * pp) + j0;
            *reinterpret_cast<__half2*>(sm + Sm::T1H + sw128_offset(rr, cc * 2)) = __floats2half2_rn(-t0, -t1);
            if (btile) *reinterpret_cast<__half2*>(btile + BT::T + sw128_offset(rr, cc * 2)) = __floats2half2_rn(-t0, -t1);
            put_t(rr, cc, -t0);
            put_t(rr, cc + 1, -t1);
        }
        // level 2: X = A_L2 T1, Y = T1 X; T[32:64, 0:32] = -Y[32:64, 0:32]
        if (!level_mma(Sm::AH2, Sm::T1H)) return false;
        // AF, XF, AH2 and DF are dead: the next item's log-decay boxes past V come in
        if (tid == kCopyThread && nc >= 0) issue_la(nh, ntok0, it + 1, true);
        store_x(Sm::XH);
        if (!level_mma(Sm::T1H, Sm::XH)) return false;
        if (row >= 32 && row < 64 && hc == 0) {
            float v[32];
            tmem_ld32_sync(tmem + lane_base, v);
#pragma unroll
            for (int i8 = 0; i8 < 4; ++i8) {
                __align__(16) __half tb[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) tb[e] = __float2half_rn(-v[8 * i8 + e] * s_beta[8 * i8 + e]);
                *reinterpret_cast<uint4*>(sm + Sm::TPV + sw128_offset(row, 16 * i8)) = *reinterpret_cast<const uint4*>(tb);
                if (btile) {
                    __align__(16) __half tt[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) tt[e] = __float2half_rn(-v[8 * i8 + e]);
                    *reinterpret_cast<uint4*>(btile + BT::T + sw128_offset(row, 16 * i8)) = *reinterpret_cast<const uint4*>(tt);
                }
            }
        }

        // ---- v: bf16 -> fp16 in place in VT, 8 values per thread and step
        ok = (!FUSED && tid != 0) || mbar_wait_cycles(&bar_v, it & 1, wait_cap);
        if (__syncthreads_or(!ok)) return false;
        v_done = it + 1;
        for (int item = tid; item < kChunk * (DV / 8); item += 256) {
            const int r = item / (DV / 8), j8 = (item - r * (DV / 8)) * 8;
            const uint32_t o = Sm::VT + (j8 >> 6) * Sm::TILE + sw128_offset(r, (j8 & 63) * 2);
            uint4 raw = *reinterpret_cast<const uint4*>(sm + o);
            if (r >= L) raw = make_uint4(0, 0, 0, 0);
            const __nv_bfloat162* vb = reinterpret_cast<const __nv_bfloat162*>(&raw);
            __align__(16) __half2 vh[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 x = __bfloat1622float2(vb[e]);
                range_max = fmaxf(range_max, fmaxf(fabsf(x.x), fabsf(x.y)));
                vh[e] = __floats2half2_rn(x.x, x.y);
            }
            *reinterpret_cast<uint4*>(sm + o) = *reinterpret_cast<const uint4*>(vh);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        if (btile && tid == kCopyThread) {   // backward mode: the fp16 V is final in VT
            bulk_store(btile + BT::V, sm + Sm::VT, (DV / 64) * Sm::TILE);
            bulk_store_commit();
            stored = true;
        }
        // ---- MMA2 (fp16): [T diag(beta); *] K~ -> D2[0, DK), [T diag(beta); *] V -> D2[DK, DK + DV)
        //      (the operand's rows 64..127 are KT's first 8 KB; their products are never read)
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idw = instr_desc(kFmtF16, 128, DK, false, true);
            constexpr uint32_t idu = instr_desc(kFmtF16, 128, DV, false, true);
            const uint32_t a0 = smem_u32(sm + Sm::TPV), bk = smem_u32(sm + Sm::KT), bv = smem_u32(sm + Sm::VT);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_f16(D2, smem_desc(a0 + ks * 32, 16, 1024, kLayoutSW128),
                        smem_desc(bk + ks * 2048, Sm::TILE, 1024, kLayoutSW128), idw, ks != 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_f16(D2 + DK, smem_desc(a0 + ks * 32, 16, 1024, kLayoutSW128),
                        smem_desc(bv + ks * 2048, Sm::TILE, 1024, kLayoutSW128), idu, ks != 0);
            mma_commit(&bar_mma);
        }
        mma_pending = 1;
        ok = (!FUSED && tid != 0) || mbar_wait_cycles(&bar_mma, mma_phase, wait_cap);
        if (__syncthreads_or(!ok)) return false;
        mma_phase ^= 1;
        mma_pending = 0;
        tc_fence_after();
        // KT and V are free: the rest of the next item's inputs come in behind the write-out
        if (tid == kCopyThread && nc >= 0) {
            if (btile) bulk_store_wait_read();   // the K~ / V tile stores have read KT and VT
            issue_k(nh, ntok0);
            issue_la(nh, ntok0, it + 1, false);
        }

        // ---- W and U0 (rows 0..63): fp16 into the OPB staging tiles (record
        //      layout), then one bulk store per tile; warps 0, 1, 4, 5 (TMEM
        //      lanes 0..63) take alternate 32-column chunks
        if ((warp & 3) < 2) {
            const int r = row;
#pragma unroll
            for (int cb = hc; cb < (DK + DV) / 32; cb += 2) {
                float v[32];
                tmem_ld32_sync(D2 + lane_base + 32 * cb, v);
#pragma unroll
                for (int i8 = 0; i8 < 4; ++i8) {
                    __align__(16) __half hv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        range_max = fmaxf(range_max, fabsf(v[8 * i8 + e]));
                        hv[e] = __float2half_rn(v[8 * i8 + e]);
                    }
                    const int col = 32 * cb + 8 * i8;   // W tiles then U0 tiles, 64 columns each
                    uint32_t dst;
                    if constexpr (FUSED)   // W: rows 0..63 of the [W; Q~] operand; U0 on its own
                        dst = col < DK ? Sm::FWQ + (uint32_t)(col >> 6) * 16384 + sw128_offset(r, (col & 63) * 2)
                                       : Sm::FU0 + h_off(r, col - DK, Sm::TILE);
                    else
                        dst = Sm::OPB + h_off(r, col, Sm::TILE);
                    *reinterpret_cast<uint4*>(sm + dst) = *reinterpret_cast<const uint4*>(hv);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();   // D2 is read; the staging tiles (or the state step's operands) are complete
        if constexpr (!FUSED) {
            if (tid == kCopyThread) {
#pragma unroll
                for (int b = 0; b < DK / 64; ++b)   // W: rows 0..63 of each WQ tile
                    bulk_store(rec + R::WQ + b * 16384, sm + Sm::OPB + b * Sm::TILE, Sm::TILE);
                bulk_store(rec + R::U0, sm + Sm::OPB + (DK / 64) * Sm::TILE, (DV / 64) * Sm::TILE);
                bulk_store_commit();
            }
        }
        ++it;
        return true;
    };

    if constexpr (!FUSED) {
        // ---- split form: items (chunk, head) w = blockIdx.x + i gridDim.x; the
        //      records go to the workspace for the inter-chunk kernel
        if (tid == kCopyThread) issue_in(blockIdx.x / H, blockIdx.x % H, 0);
        in_issued = 1;
        load_beta(blockIdx.x / H, blockIdx.x % H);
        for (int w = blockIdx.x; w < total; w += gridDim.x) {
            const int c = w / H, h = w - c * H;
            int seq, tok0, L;
            map.locate(c, seq, tok0, L);
            const int wn = w + gridDim.x;
            if (!run_item(c, h, tok0, L, wn < total ? wn / H : -1, wn < total ? wn % H : 0)) { aborted = true; break; }
        }
    } else {
        // ---- fused form: whole (sequence, head) pairs, claimed longest first;
        //      after each chunk's intra-chunk phases the state step consumes the
        //      chunk's operands from shared memory (no records), with the fp32
        //      state resident in TMEM for the whole sequence
        constexpr int CPT = DV / 2;                       // state columns per thread
        const uint32_t cb = (uint32_t)(CPT * hc);
        int* s_pair = reinterpret_cast<int*>(sm + Sm::PAIR);
        auto ld_cols = [&](uint32_t taddr, float (&v)[CPT]) {
#pragma unroll
            for (int c0 = 0; c0 < CPT; c0 += 32) {
                float t[32];
                tmem_ld32_sync(taddr + c0, t);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[c0 + i] = t[i];
            }
        };
        auto st_cols = [&](uint32_t taddr, const float (&v)[CPT]) {
#pragma unroll
            for (int c0 = 0; c0 < CPT; c0 += 32) {
                float t[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) t[i] = v[c0 + i];
                tmem_st32_sync(taddr + c0, t);
            }
        };
        // fp16 copy of this thread's state columns (row = key channel): MMA3's B operand
        auto put_s16 = [&](const float (&v)[CPT]) {
#pragma unroll
            for (int i8 = 0; i8 < CPT / 8; ++i8) {
                const uint32_t col = cb + 8 * i8;
                __align__(16) __half2 hv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float x0 = v[8 * i8 + 2 * e], x1 = v[8 * i8 + 2 * e + 1];
                    range_max = fmaxf(range_max, fmaxf(fabsf(x0), fabsf(x1)));
                    hv[e] = __floats2half2_rn(x0, x1);
                }
                *reinterpret_cast<uint4*>(sm + Sm::S16 + (col >> 6) * 16384 + sw128_offset(row, (col & 63) * 2)) =
                    *reinterpret_cast<const uint4*>(hv);
            }
        };
        // one chunk of the state recurrence, on the chunk's on-chip operands:
        //   U = U0 - W S,  O = d_k^{-1/2} (Q~ S + P U),  S <- Diag(gamma_C) S + K^^T U
        auto state_step = [&](int tok0, int L, int h) -> bool {
            if (tid == 0) {   // MMA3: [W; Q~] S -> R3
                tc_fence_after();
                constexpr uint32_t idesc = instr_desc(kFmtF16, 128, DV, false, true);
                const uint32_t a0 = smem_u32(sm + Sm::FWQ), b0 = smem_u32(sm + Sm::S16);
#pragma unroll
                for (int kb = 0; kb < DK / 64; ++kb)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_f16(R3, smem_desc(a0 + kb * 16384 + ks * 32, 16, 1024, kLayoutSW128),
                                smem_desc(b0 + kb * 8192 + ks * 2048, 16384, 1024, kLayoutSW128), idesc, (kb | ks) != 0);
                mma_commit(&bar_mma);
            }
            mma_pending = 1;
            if (row < DK) {   // S <- Diag(gamma_C) S while MMA3 reads the fp16 copy
                const float gcv = reinterpret_cast<const float*>(sm + Sm::FGC)[row];
                float v[CPT];
                ld_cols(SACC + lane_base + cb, v);
#pragma unroll
                for (int i = 0; i < CPT; ++i) v[i] *= gcv;
                st_cols(SACC + lane_base + cb, v);
            }
            bool ok = mbar_wait_cycles(&bar_mma, mma_phase, wait_cap);
            if (__syncthreads_or(!ok)) return false;
            mma_phase ^= 1;
            mma_pending = 0;
            tc_fence_after();
            if (row < 64) {   // U = U0 - W S (rows = tokens) -> U16
                float v[CPT];
                ld_cols(R3 + lane_base + cb, v);
#pragma unroll
                for (int i8 = 0; i8 < CPT / 8; ++i8) {
                    const uint32_t off = h_off(row, cb + 8 * i8, Sm::TILE);
                    const uint4 u0raw = *reinterpret_cast<const uint4*>(sm + Sm::FU0 + off);
                    const __half2* u0 = reinterpret_cast<const __half2*>(&u0raw);
                    __align__(16) __half2 hv[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 u0f = __half22float2(u0[e]);
                        const float ua = u0f.x - v[8 * i8 + 2 * e], ub = u0f.y - v[8 * i8 + 2 * e + 1];
                        range_max = fmaxf(range_max, fmaxf(fabsf(ua), fabsf(ub)));
                        hv[e] = __floats2half2_rn(ua, ub);
                    }
                    *reinterpret_cast<uint4*>(sm + Sm::U16 + off) = *reinterpret_cast<const uint4*>(hv);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {   // MMA4: [*; P] U += R3;  MMA5: K^^T U += S
                tc_fence_after();
                constexpr uint32_t idesc = instr_desc(kFmtF16, 128, DV, false, true);
                constexpr uint32_t idesc_t = instr_desc(kFmtF16, 128, DV, true, true);
                const uint32_t pa = smem_u32(sm + Sm::FP) - 8192, ub = smem_u32(sm + Sm::U16);
                const uint32_t ka = smem_u32(sm + Sm::FKH);
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
            ok = mbar_wait_cycles(&bar_mma, mma_phase, wait_cap);
            if (__syncthreads_or(!ok)) return false;
            mma_phase ^= 1;
            mma_pending = 0;
            tc_fence_after();
            if (row >= 64) {   // output rows
                const int r = row - 64;
                float v[CPT];
                ld_cols(R3 + lane_base + cb, v);
                if (r < L) {
                    __nv_bfloat16* dst = o + ((size_t)(tok0 + r) * H + h) * DV + cb;
#pragma unroll
                    for (int i8 = 0; i8 < CPT / 8; ++i8) {
                        __align__(16) __nv_bfloat162 bv[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            bv[e] = __floats2bfloat162_rn(scale * v[8 * i8 + 2 * e], scale * v[8 * i8 + 2 * e + 1]);
                        *reinterpret_cast<uint4*>(dst + 8 * i8) = *reinterpret_cast<const uint4*>(bv);
                    }
                }
            }
            if (row < DK) {   // the next chunk's fp16 state operand
                float v[CPT];
                ld_cols(SACC + lane_base + cb, v);
                put_s16(v);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            return true;
        };

        const int num_pairs = map.num_seqs * H;
        for (;;) {
            if (tid == 0) *s_pair = atomicAdd(&hdr->next_pair, 1);
            __syncthreads();
            const int p = *s_pair;
            __syncthreads();
            if (p >= num_pairs) break;
            const int si = p / H, h = p - si * H;
            const int s = seq_order ? seq_order[si] : si;
            const int first = map.seq_first_chunk(s), nch = map.seq_num_chunks(s);
            const int tb = map.seq_token_begin(s), te = map.seq_token_end(s);
            const size_t soff = ((size_t)s * H + h) * DK * DV;
            if (nch <= 0) {   // empty sequence: the state passes through
                if (final_state)
                    for (int i = tid; i < DK * DV; i += 256) final_state[soff + i] = initial_state ? initial_state[soff + i] : 0.f;
                continue;
            }
            if (tid == kCopyThread) issue_in(first, h, it);
            in_issued = it + 1;
            load_beta(first, h);
            if (row < DK) {   // initial state -> TMEM (fp32) and its fp16 operand copy
                float v[CPT];
#pragma unroll
                for (int i = 0; i < CPT; i += 4) {
                    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (initial_state) x = *reinterpret_cast<const float4*>(initial_state + soff + (size_t)row * DV + cb + i);
                    v[i] = x.x; v[i + 1] = x.y; v[i + 2] = x.z; v[i + 3] = x.w;
                }
                st_cols(SACC + lane_base + cb, v);
                put_s16(v);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            for (int j = 0; j < nch; ++j) {
                const int tok0 = tb + j * kChunk, L = min(kChunk, te - tok0);
                if (!run_item(first + j, h, tok0, L, j + 1 < nch ? first + j + 1 : -1, h)) { aborted = true; break; }
                if (!state_step(tok0, L, h)) { aborted = true; break; }
            }
            if (aborted) break;
            if (final_state && row < DK) {
                float v[CPT];
                ld_cols(SACC + lane_base + cb, v);
                float* dst = final_state + soff + (size_t)row * DV + cb;
#pragma unroll
                for (int i = 0; i < CPT; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
            }
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
        }
    }

    if (aborted) {
        if (tid == 0) flag_error(hdr, kStatusTimeout);
        // let this CTA's own copies and MMAs finish (bounded) before its memory goes away
        if (tid == 0) {
            for (int j = in_done; j < in_issued; ++j) (void)mbar_wait_cycles(&bar_in, j & 1, wait_cap / 4);
            for (int j = v_done; j < v_issued; ++j) (void)mbar_wait_cycles(&bar_v, j & 1, wait_cap / 4);
            if (mma_pending) (void)mbar_wait_cycles(&bar_mma, mma_phase, wait_cap);
        }
    }
    if (tid == kCopyThread && stored) bulk_store_wait_all();
    if (range_max > kF16Limit) flag_error(hdr, kStatusRange);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// Packed sequences ordered longest first (ties by index), the order in which the
// forward's per-sequence CTAs are started (the fused pass's pair queue, the
// inter-chunk kernel's grid), so that the longest chains do not start last:
// order[rank(s)] = s.  One block; beyond 16384 sequences the order is left as
// given.
__global__ void __launch_bounds__(1024)
seq_order_kernel(const WsHeader* hdr, const int32_t* __restrict__ cu, int N, int* __restrict__ order)
{
    if (hdr->status != kStatusOk) return;
    for (int s = threadIdx.x; s < N; s += blockDim.x) {
        int rank = s;
        if (N <= 16384) {
            const int len = cu[s + 1] - cu[s];
            rank = 0;
            for (int t = 0; t < N; ++t) {
                const int lt = cu[t + 1] - cu[t];
                rank += (lt > len) || (lt == len && t < s);
            }
        }
        order[rank] = s;
    }
}

template <int DK, int DV, bool FUSED>
cudaError_t launch_intra_fwd_tc_t(const ChunkArgs& a) {
    if (a.max_chunks == 0 && !FUSED) return cudaSuccess;
    const int ntok = a.cu_seqlens ? a.T : a.B * a.T;
    CUtensorMap mk, mv, mq, mla;
    memset(&mk, 0, sizeof(mk));
    memset(&mv, 0, sizeof(mv));
    memset(&mq, 0, sizeof(mq));
    memset(&mla, 0, sizeof(mla));
    if (ntok > 0 &&
        (!make_map(&mk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, a.H, ntok, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
         !make_map(&mv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DV, a.H, ntok, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
         !make_map(&mq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, a.H, ntok, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
         (a.gate == kGateChannel &&
          !make_map(&mla, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, DK, a.H, ntok, 32, CU_TENSOR_MAP_SWIZZLE_128B))))
        return cudaErrorInvalidValue;
    ChunkMap map{a.cu_seqlens, a.chunk_offsets, a.num_seqs, a.T, a.fixed_chunks_per_seq};
    // backward mode (the split form with backward tiles) is its own instance, so
    // the plain forward carries none of its stores
    const bool bwd = !FUSED && a.bwd_tiles != nullptr;
    auto kern = a.gate == kGateChannel ? intra_chunk_fwd_tc_kernel<DK, DV, kGateChannel, FUSED, false>
              : a.gate == kGateHead    ? intra_chunk_fwd_tc_kernel<DK, DV, kGateHead, FUSED, false>
                                       : intra_chunk_fwd_tc_kernel<DK, DV, kGateNone, FUSED, false>;
    if constexpr (!FUSED) {
        if (bwd)
            kern = a.gate == kGateChannel ? intra_chunk_fwd_tc_kernel<DK, DV, kGateChannel, false, true>
                 : a.gate == kGateHead    ? intra_chunk_fwd_tc_kernel<DK, DV, kGateHead, false, true>
                                          : intra_chunk_fwd_tc_kernel<DK, DV, kGateNone, false, true>;
    }
    const int smem = (int)K1fSmem<DK, DV, FUSED>::TOTAL;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    unsigned grid;
    const int* order = a.seq_order;   // pairs claimed longest first (null: in order)
    if constexpr (FUSED) {
        const size_t pairs = (size_t)a.num_seqs * a.H;
        grid = (unsigned)(pairs < (size_t)sms ? pairs : (size_t)sms);   // one resident per SM
        if (grid == 0) return cudaSuccess;
    } else {
        const size_t items = a.max_chunks * (size_t)a.H;   // upper bound; the kernel reads the exact count
        const size_t ctas = 2 * (size_t)sms;               // two resident per SM
        grid = (unsigned)(items < ctas ? items : ctas);
    }
    kern<<<grid, 256, smem, a.stream>>>(mk, mv, mq, mla, a.log_alpha, a.beta, map,
                                        static_cast<WsHeader*>(a.ws_header),
                                        static_cast<unsigned char*>(a.records), a.H, a.max_chunks,
                                        a.wait_cap > 0 ? a.wait_cap : kWaitCycles, a.debug_drop_copy,
                                        a.initial_state, a.final_state, static_cast<__nv_bfloat16*>(a.o), a.scale,
                                        order, bwd ? static_cast<unsigned char*>(a.bwd_tiles) : nullptr,
                                        bwd ? a.bwd_flags : nullptr);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_intra_fwd_tc(const ChunkArgs& a) {
    if (a.dk == 128 && a.dv == 128) return launch_intra_fwd_tc_t<128, 128, false>(a);
    if (a.dk == 128 && a.dv == 64) return launch_intra_fwd_tc_t<128, 64, false>(a);
    if (a.dk == 64 && a.dv == 128) return launch_intra_fwd_tc_t<64, 128, false>(a);
    if (a.dk == 64 && a.dv == 64) return launch_intra_fwd_tc_t<64, 64, false>(a);
    return cudaErrorInvalidValue;
}

cudaError_t launch_chunk_seq_order(const ChunkArgs& a) {
    if (!a.seq_order || !a.cu_seqlens || a.num_seqs <= 1) return cudaSuccess;
    seq_order_kernel<<<1, 1024, 0, a.stream>>>(static_cast<WsHeader*>(a.ws_header), a.cu_seqlens, a.num_seqs,
                                               a.seq_order);
    return cudaGetLastError();
}

cudaError_t launch_chunk_fused_tc(const ChunkArgs& a) {
    if (a.num_seqs == 0) return cudaSuccess;
    if (a.dk == 128 && a.dv == 128) return launch_intra_fwd_tc_t<128, 128, true>(a);
    if (a.dk == 128 && a.dv == 64) return launch_intra_fwd_tc_t<128, 64, true>(a);
    if (a.dk == 64 && a.dv == 128) return launch_intra_fwd_tc_t<64, 128, true>(a);
    if (a.dk == 64 && a.dv == 64) return launch_intra_fwd_tc_t<64, 64, true>(a);
    return cudaErrorInvalidValue;
}

}  // namespace kda
