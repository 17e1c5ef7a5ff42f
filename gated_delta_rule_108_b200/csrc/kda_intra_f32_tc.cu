// kda_intra_f32_tc.cu -- the forward intra-chunk kernel for fp32 inputs on the
// sm_100a tensor cores.
//
// The same chunk algebra as the bf16 intra-chunk kernel (kda_intra_tc.cu; the
// chunk-wise parallel form of kongchang.com "Kimi Delta Attention详解", section
// "硬件效率的优化策略", from the daiw.net update equation, section "KDA 的更新式"),
// with every product in split tf32 so that fp32 inputs keep fp32-level
// accuracy: each operand x is cut into hi = x with its low 13 mantissa bits
// cleared (exact in tf32) and lo = x - hi (exact in fp32), and a product is
// hi.hi + hi.lo + lo.hi with fp32 accumulation in tensor memory.  Per (chunk,
// head) item, with g the cumulative log-decay (base 2) and g_m the middle token's:
//
//   [A; P] = [K~m; Q~m] K-m^T     A operand (hi, lo) in TMEM, K-m (hi, lo) in smem
//   T = (I + A)^{-1}              16 x 16 blocks on CUDA cores, fp32
//   [W | U0] = T diag(beta) [K~ | V]   T diag(beta) (hi, lo) in TMEM, K~^T, V^T in smem
//
// and writes the fp32 record (F32TcRec) that the fp32 tensor-core inter-chunk
// kernel reads.
// Chunks whose decay is too strong for the split factors e^{+-(g - g_m)} form
// A and P exactly on CUDA cores (every exponent <= 0), as the other kernels do.
//
// tf32 operands must be K-major (contiguous along the contraction index).  The
// element pass runs one thread per token row, so the operands contracted over
// tokens (K~, V for W and U0) are written transposed, 32 consecutive tokens of
// a warp filling one 128-byte row: no bank conflicts either way.
//
// One CTA (8 warps) per SM, persistent over the (chunk, head) items.  The only
// mbarrier is the MMA completion; every wait is bounded and a CTA that gives up
// records KDA_ERR_TIMEOUT, waits (bounded) for its MMAs, frees its tensor
// memory and returns.
#include "kda_common.cuh"
#include "kda_launch.h"
#include "kda_tc_common.cuh"
#include "ptx.cuh"

namespace kda {
namespace {

using namespace ptx;

// x = hi + lo: hi keeps the sign, exponent and top 10 mantissa bits (a tf32
// value, used by the tensor core as is); lo = x - hi is exact in fp32 and
// below 2^-10 |x|, so the tensor core's own cut of lo costs < 2^-20 |x|.
__device__ __forceinline__ void split_tf32(float x, float& hi, float& lo) {
    hi = __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
    lo = x - hi;
}

template <int DK, int DV>
struct F32K1Smem {
    static constexpr int LDK = DK + 4;                  // padded row strides (floats): conflict-free
    static constexpr int LDV = DV + 4;                  // 16-byte accesses by one thread per row
    static constexpr int LDA = kChunk + 1;              // and scalar ones along a column
    // BIG, reused through an item:
    //   item start: this item's k and q rows ([64][DK] each, 16-byte chunks XOR-swizzled by row
    //     within 128 bytes), copied in at the end of the previous item
    //   element pass .. MMA1: K-m (hi | lo) at KB, token-major, K = channel, DK/32 tiles of
    //     64 rows x 128 B (strong-decay chunks: raw k and q [64][DK] there instead), and
    //     K~^T (hi | lo) at KTT, channel-major, 2 tiles (tokens 0..31, 32..63) of DK rows x 128 B
    //   after MMA1: T and its partial products, then V^T (hi | lo) at KB, 2 tiles of
    //     DV rows x 128 B, until MMA2
    //   after MMA2: the next item's k and q
    static constexpr uint32_t KB = 0;
    static constexpr uint32_t KB_BYTES = (DK > DV ? DK : DV) * 512u;
    static constexpr uint32_t KTT = KB + KB_BYTES;
    static constexpr uint32_t KTT_BYTES = DK * 512u;
    static constexpr uint32_t BIG_BYTES = KB_BYTES + KTT_BYTES;
    static constexpr uint32_t KQ_Q = 64u * DK * 4u;      // q staging, after k's
    static constexpr uint32_t G = BIG_BYTES;             // log-decay (copied in early), then g (base 2): [64][LDK]
    static constexpr uint32_t AM = G + 64u * LDK * 4u;   // A (beta-scaled, strictly lower), then P [64][LDA]
    static constexpr uint32_t VS = AM + 64u * LDA * 4u;  // v [64][LDV] (copied in at the item's start)
    // after MMA2, over G, AM and VS: W [64][LDK] and U0 [64][LDV], staged for coalesced stores
    static constexpr uint32_t WS = G, US = G + 64u * LDK * 4u;
    static constexpr uint32_t BETA = VS + 64u * LDV * 4u;
    static constexpr uint32_t LAH = BETA + 256u;         // per-head log-decay [64]
    static constexpr uint32_t END = LAH + 256u;
    static_assert(KB % 1024 == 0 && KTT % 1024 == 0, "operand tiles are 1024-byte aligned");
    static_assert(2u * 64u * DK * 4u <= KB_BYTES, "k, q staging lies clear of K~^T");
    static_assert(US + 64u * LDV * 4u <= VS + 64u * LDV * 4u, "W, U0 staging fits");
    static_assert(64u * LDA * 4u + 3u * 16u * 17u * 4u <= KB_BYTES, "T and its partial products fit in K-m's space");
    static_assert(END + 1024 <= 232448, "shared memory");
};

template <int DK, int DV, int GATE>
__global__ void __launch_bounds__(256, 1)
intra_chunk_f32_tc_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                          const float* __restrict__ log_alpha, const float* __restrict__ beta, ChunkMap map,
                          WsHeader* hdr, float* __restrict__ records, int H, size_t max_chunks)
{
    using Sm = F32K1Smem<DK, DV>;
    using R = F32TcRec<DK, DV>;
    constexpr int LDK = Sm::LDK, LDV = Sm::LDV, LDA = Sm::LDA;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bar_mma;
    __shared__ uint32_t s_tmem;

    if (hdr->status != kStatusOk) return;
    const int total = hdr->num_chunks * H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = 32 * (warp & 3) + lane;   // TMEM lane: 0..63 K rows, 64..127 Q rows
    const int hc = warp >> 2;                 // column half
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const bool is_k = row < 64;
    const int r_el = is_k ? row : row - 64;   // this thread's token row in the element pass
    float* g = reinterpret_cast<float*>(sm + Sm::G);
    float* am = reinterpret_cast<float*>(sm + Sm::AM);
    float* s_beta = reinterpret_cast<float*>(sm + Sm::BETA);
    float* s_lah = reinterpret_cast<float*>(sm + Sm::LAH);
    const size_t rowk = (size_t)H * DK, rowv = (size_t)H * DV;

    if (tid == 0) {
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
    const uint32_t A1 = tmem;                  // [K~m; Q~m] hi at +0, lo at +DK (128 lanes x DK)
    const uint32_t D1 = tmem + 2 * DK;         // [A; P] (128 lanes x 64)
    const uint32_t A2 = tmem + 2 * DK + 64;    // T diag(beta) hi at +0, lo at +64 (lanes 0..63)
    const uint32_t D2 = tmem;                  // [W | U0] (lanes 0..63 x (DK + DV)), after MMA1
    static_assert(DK + DV <= 2 * DK + 64, "W | U0 must end before T diag(beta)");

    bool aborted = false;
    uint32_t mma_phase = 0;
    int mma_pending = 0;
    auto wait_mma = [&]() -> bool {
        const bool ok = mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        if (__syncthreads_or(!ok)) return false;
        mma_phase ^= 1;
        mma_pending = 0;
        tc_fence_after();
        return true;
    };
    // 16-byte cp.async of `n16` granules of 64 rows (row r: n16 / 64 granules from
    // src + (tok0 + r) * stride) into padded smem rows; rows past L are zero-filled
    auto copy_rows = [&](float* dst, int ld, const float* src, size_t stride, int per_row, int tok0, int L) {
        for (int idx = tid; idx < 64 * per_row; idx += 256) {
            const int r = idx / per_row, c4 = (idx - r * per_row) * 4;
            cp_async16(dst + r * ld + c4, src + (size_t)(tok0 + (r < L ? r : 0)) * stride + c4, r < L ? 16u : 0u);
        }
    };
    // float offset of the 16-byte chunk holding channels [4 lc, 4 lc + 4) of row r in the
    // staged k / q (chunks XOR-swizzled by r mod 8 within each 128-byte group)
    auto kq_off = [](int r, int lc) { return r * DK + (((lc & ~7) | ((lc & 7) ^ (r & 7))) << 2); };
    auto locate = [&](int w, int& h, int& tok0, int& L) {
        const int c = w / H;
        h = w - c * H;
        int seq;
        map.locate(c, seq, tok0, L);
    };
    // the log-decay tile of item w (per-channel gate) into G; its v into VS
    auto prefetch_la = [&](int w) {
        int h, tok0, L;
        locate(w, h, tok0, L);
        if constexpr (GATE == kGateChannel) copy_rows(g, LDK, log_alpha + (size_t)h * DK, rowk, DK / 4, tok0, L);
        cp_async_commit();
    };
    auto prefetch_v = [&](int w) {
        int h, tok0, L;
        locate(w, h, tok0, L);
        copy_rows(reinterpret_cast<float*>(sm + Sm::VS), LDV, v + (size_t)h * DV, rowv, DV / 4, tok0, L);
        cp_async_commit();
    };
    // k and q of item w into BIG
    auto prefetch_kq = [&](int w) {
        int h, tok0, L;
        locate(w, h, tok0, L);
        for (int idx = tid; idx < 64 * (DK / 4); idx += 256) {
            const int r = idx / (DK / 4), lc = idx - r * (DK / 4);
            const size_t so = (size_t)(tok0 + (r < L ? r : 0)) * rowk + (size_t)h * DK + 4 * lc;
            const uint32_t nb = r < L ? 16u : 0u;
            cp_async16(reinterpret_cast<float*>(sm) + kq_off(r, lc), k + so, nb);
            cp_async16(reinterpret_cast<float*>(sm + Sm::KQ_Q) + kq_off(r, lc), q + so, nb);
        }
        cp_async_commit();
    };
    if ((int)blockIdx.x < total) {
        prefetch_kq(blockIdx.x);
        prefetch_la(blockIdx.x);
    }

    for (int w = blockIdx.x; w < total; w += gridDim.x) {
        const int c = w / H, h = w - c * H;
        int seq, tok0, L;
        map.locate(c, seq, tok0, L);
        float* rec = records + ((size_t)h * max_chunks + c) * R::FLOATS;
        const bool has_next = w + (int)gridDim.x < total;

        // ---- beta, the per-head log-decay; the copied tiles; this thread's k or
        //      q row (channels [hc DK/2, hc DK/2 + DK/2)) into registers
        if constexpr (GATE != kGateChannel) {
            if (tid >= 192) {
                const int r = tid - 192;
                s_lah[r] = (GATE == kGateHead && r < L) ? log_alpha[(size_t)(tok0 + r) * H + h] : 0.f;
            }
        }
        if (tid >= 128 && tid < 192) {
            const int r = tid - 128;
            s_beta[r] = r < L ? beta[(size_t)(tok0 + r) * H + h] : 0.f;
        }
        prefetch_v(w);        // lands during the element pass and MMA1
        cp_async_wait<1>();   // k, q and the log-decay tile
        __syncthreads();
        float xa[DK / 2];
        {
            const float* src = reinterpret_cast<const float*>(sm + (is_k ? 0u : Sm::KQ_Q));
#pragma unroll
            for (int j = 0; j < DK / 2; j += 4) {
                const float4 a = *reinterpret_cast<const float4*>(src + kq_off(r_el, (hc * (DK / 2) + j) >> 2));
                xa[j] = a.x; xa[j + 1] = a.y; xa[j + 2] = a.z; xa[j + 3] = a.w;
            }
        }
        // ---- cumulative log-decay per channel, base 2 (rows past L add 0): each
        //      channel's 64 rows in 256 / DK parts, scanned locally, then offset
        {
            constexpr int NP = 256 / DK, RP = 64 / NP;
            const int ch = tid % DK, part = tid / DK;
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < RP; ++i) {
                const int r = part * RP + i;
                const float la = GATE == kGateChannel ? g[r * LDK + ch] : s_lah[r];
                acc += la * kLog2e;
                g[r * LDK + ch] = acc;
            }
            __syncthreads();
            float off = 0.f;
#pragma unroll
            for (int p = 0; p < NP - 1; ++p)
                if (p < part) off += g[((p + 1) * RP - 1) * LDK + ch];
            __syncthreads();
            if (part > 0) {
#pragma unroll
                for (int i = 0; i < RP; ++i) g[(part * RP + i) * LDK + ch] += off;
            }
        }
        __syncthreads();
        const float* gmid = g + ((L - 1) >> 1) * LDK;
        const float* gend = g + (L - 1) * LDK;
        bool wide = false;
        if (tid < DK) wide = fmaxf(g[tid] - gmid[tid], gmid[tid] - gend[tid]) > kMaxSplitExponent2;
        // ---- record Q~ = q e^{g} (rows 64..127 of WQ; coalesced, from the staged q)
        //      and gamma_C
        {
            const float* qs = reinterpret_cast<const float*>(sm + Sm::KQ_Q);
#pragma unroll 4
            for (int idx = tid; idx < 64 * (DK / 4); idx += 256) {
                const int r = idx / (DK / 4), c4 = (idx - r * (DK / 4)) * 4;
                const float4 qq = *reinterpret_cast<const float4*>(qs + kq_off(r, c4 >> 2));
                const float4 gg = *reinterpret_cast<const float4*>(g + r * LDK + c4);
                *reinterpret_cast<float4*>(rec + R::WQ + (size_t)(64 + r) * DK + c4) =
                    make_float4(qq.x * ex2_approx(gg.x), qq.y * ex2_approx(gg.y), qq.z * ex2_approx(gg.z),
                                qq.w * ex2_approx(gg.w));
            }
            if (tid < DK) rec[R::GC + tid] = ex2_approx(gend[tid]);
        }
        // ---- from the staged k, by all threads (warp = 32 consecutive tokens of one
        //      quarter of the channels): the record K^ = k e^{g_{L-1} - g} transposed
        //      and K~ = k e^{g} -> K~^T (hi | lo), MMA2's B operand; a warp fills 128
        //      contiguous bytes of a channel row in both
        {
            const float* ks = reinterpret_cast<const float*>(sm);
            const int r = 32 * (warp & 1) + lane, cq = warp >> 1;
            const uint32_t ktt_lo = 2u * DK * 128u;
#pragma unroll 2
            for (int c4 = cq * (DK / 4); c4 < (cq + 1) * (DK / 4); c4 += 4) {
                const float4 kk = *reinterpret_cast<const float4*>(ks + kq_off(r, c4 >> 2));
                const float4 gg = *reinterpret_cast<const float4*>(g + r * LDK + c4);
                const float4 ge = *reinterpret_cast<const float4*>(gend + c4);
                const float kv[4] = {kk.x, kk.y, kk.z, kk.w}, gv[4] = {gg.x, gg.y, gg.z, gg.w};
                const float gev[4] = {ge.x, ge.y, ge.z, ge.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    rec[R::KHT + (size_t)(c4 + e) * kChunk + r] = kv[e] * ex2_approx(gev[e] - gv[e]);
                    float hi, lo;
                    split_tf32(kv[e] * ex2_approx(gv[e]), hi, lo);
                    const uint32_t off = (uint32_t)(r >> 5) * (DK * 128u) + sw128_offset(c4 + e, (r & 31) * 4);
                    *reinterpret_cast<float*>(sm + Sm::KTT + off) = hi;
                    *reinterpret_cast<float*>(sm + Sm::KTT + ktt_lo + off) = lo;
                }
            }
        }
        const bool strong = __syncthreads_or(wide);   // k and q are read: their space is free

        // ---- element pass: thread = token row (K rows on lanes 0..63, Q rows on
        //      64..127), channels [hc DK/2, hc DK/2 + DK/2) in groups of 8
        {
            const int r = r_el;
            float* kraw = reinterpret_cast<float*>(sm + Sm::KB);   // strong: raw k, then raw q
            const uint32_t kb_lo = (DK / 32) * 8192u;
#pragma unroll
            for (int j = 0; j < DK / 2; j += 8) {
                const int c8 = hc * (DK / 2) + j;
                float x[8], gr[8], gm[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    x[e] = xa[j + e];
                    gr[e] = g[r * LDK + c8 + e];
                    gm[e] = gmid[c8 + e];
                }
                if (!strong) {
                    // K~m = k e^{g - g_m} | Q~m = q e^{g - g_m} -> TMEM (hi | lo), MMA1's A operand
                    uint32_t th[8], tl[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        float hi, lo;
                        split_tf32(x[e] * ex2_approx(gr[e] - gm[e]), hi, lo);
                        th[e] = __float_as_uint(hi);
                        tl[e] = __float_as_uint(lo);
                    }
                    tmem_st8(A1 + lane_base + c8, th);
                    tmem_st8(A1 + lane_base + DK + c8, tl);
                    if (is_k) {   // K-m = k e^{g_m - g} -> smem (hi | lo), MMA1's B operand
                        __align__(16) float bh[8], bl[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) split_tf32(x[e] * ex2_approx(gm[e] - gr[e]), bh[e], bl[e]);
                        const uint32_t o0 = f_off(r, c8, 8192), o1 = f_off(r, c8 + 4, 8192);
                        *reinterpret_cast<float4*>(sm + Sm::KB + o0) = *reinterpret_cast<const float4*>(bh);
                        *reinterpret_cast<float4*>(sm + Sm::KB + o1) = *reinterpret_cast<const float4*>(bh + 4);
                        *reinterpret_cast<float4*>(sm + Sm::KB + kb_lo + o0) = *reinterpret_cast<const float4*>(bl);
                        *reinterpret_cast<float4*>(sm + Sm::KB + kb_lo + o1) = *reinterpret_cast<const float4*>(bl + 4);
                    }
                } else {   // raw k / q for the exact A and P
                    float* dst = kraw + (is_k ? 0 : 64 * DK) + r * DK + c8;
                    *reinterpret_cast<float4*>(dst) = make_float4(x[0], x[1], x[2], x[3]);
                    *reinterpret_cast<float4*>(dst + 4) = make_float4(x[4], x[5], x[6], x[7]);
                }
            }
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        if (!strong) {
            // ---- MMA1: [A; P] = [K~m; Q~m] K-m^T in split tf32 (lo terms first)
            if (tid == 0) {
                tc_fence_after();
                constexpr uint32_t idesc = instr_desc(kFmtTF32, 128, 64);
                const uint32_t b0 = smem_u32(sm + Sm::KB), b_lo = (DK / 32) * 8192u;
#pragma unroll
                for (int pass = 0; pass < 3; ++pass) {
                    const uint32_t acol = pass == 1 ? DK : 0;      // hi.lo, lo.hi, hi.hi
                    const uint32_t boff = pass == 0 ? b_lo : 0;
#pragma unroll
                    for (int kb = 0; kb < DK / 32; ++kb)
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            mma_tf32_ts(D1, A1 + acol + kb * 32 + ks * 8,
                                        smem_desc(b0 + boff + kb * 8192 + ks * 32, 16, 1024, kLayoutSW128), idesc,
                                        (pass | kb | ks) != 0);
                }
                mma_commit(&bar_mma);
            }
            mma_pending = 1;
            if (!wait_mma()) { aborted = true; break; }
            // ---- A (lanes 0..63) -> smem, beta-scaled and strictly lower
            if (is_k) {
                float vv[32];
                tmem_ld32_sync(D1 + lane_base + 32 * hc, vv);
                const float br = s_beta[row];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int i = 32 * hc + e;
                    am[row * LDA + i] = i < row ? br * vv[e] : 0.f;
                }
            }
        } else {
            // ---- exact A and P: one warp per (r, i), lanes over channels; every
            //      exponent g_r - g_i (i <= r) is <= 0
            const float* kr_ = reinterpret_cast<const float*>(sm + Sm::KB);
            const float* qr_ = kr_ + 64 * DK;
            for (int pr = warp; pr < 64 * 64; pr += 8) {
                const int r = pr >> 6, i = pr & 63;
                float sa = 0.f, sp = 0.f;
                if (i <= r && r < L) {
#pragma unroll
                    for (int c0 = 0; c0 < DK; c0 += 32) {
                        const int cc = c0 + lane;
                        const float wgt = ex2_approx(g[r * LDK + cc] - g[i * LDK + cc]);
                        const float ki = kr_[i * DK + cc];
                        sa = fmaf(kr_[r * DK + cc] * ki, wgt, sa);
                        sp = fmaf(qr_[r * DK + cc] * ki, wgt, sp);
                    }
#pragma unroll
                    for (int off = 16; off; off >>= 1) {
                        sa += __shfl_xor_sync(0xffffffffu, sa, off);
                        sp += __shfl_xor_sync(0xffffffffu, sp, off);
                    }
                }
                if (lane == 0) {
                    am[r * LDA + i] = i < r ? s_beta[r] * sa : 0.f;
                    rec[R::P + (i >> 5) * 2048 + sw128_offset(r, (i & 31) * 4) / 4] = i <= r ? sp : 0.f;
                }
            }
        }
        cp_async_wait<0>();   // v
        __syncthreads();      // A complete; K-m (or raw k, q) is dead; v has landed

        // ---- T = (I + A)^{-1}, blocked over 16 x 16 blocks (all threads, fp32, in
        //      the free K-m space): the diagonal blocks by forward substitution,
        //      then T_ij = -T_ii sum_{j <= m < i} A_im T_mj level by level
        {
            float* tt = reinterpret_cast<float*>(sm + Sm::KB);   // T [64][LDA]
            float* xs = tt + 64 * LDA;                            // [3][16][17] partial products
            if (tid < 64) {
                const int kb = tid >> 4, j = tid & 15, o0 = 16 * kb;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float acc = (r == j) ? 1.f : 0.f;
#pragma unroll
                    for (int i = 0; i < r; ++i) acc = fmaf(-am[(o0 + r) * LDA + o0 + i], x[i], acc);
                    x[r] = acc;
                    tt[(o0 + r) * LDA + o0 + j] = acc;
                }
            } else {   // zero above the diagonal blocks
                for (int idx = tid - 64; idx < 6 * 256; idx += 192) {
                    const int blk = idx >> 8, e2 = idx & 255, i = e2 >> 4, j = e2 & 15;
                    const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
                    const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
                    tt[(16 * bi + i) * LDA + 16 * bj + j] = 0.f;
                }
            }
            __syncthreads();
            const int bi = tid >> 4, bj = tid & 15;   // element of a 16 x 16 block
            // X = sum_{m = mj}^{mi - 1} A_{mi, m} T_{m, mj};  T_{mi, mj} = -T_{mi, mi} X
            auto x_part = [&](int mi, int mj, float* xo) {
                float acc = 0.f;
                for (int m = mj; m < mi; ++m)
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        acc = fmaf(am[(16 * mi + bi) * LDA + 16 * m + q], tt[(16 * m + q) * LDA + 16 * mj + bj], acc);
                xo[bi * 17 + bj] = acc;
            };
            auto t_part = [&](int mi, int mj, const float* xi) {
                float acc = 0.f;
#pragma unroll
                for (int q = 0; q < 16; ++q) acc = fmaf(tt[(16 * mi + bi) * LDA + 16 * mi + q], xi[q * 17 + bj], acc);
                tt[(16 * mi + bi) * LDA + 16 * mj + bj] = -acc;
            };
            x_part(1, 0, xs);
            x_part(2, 1, xs + 272);
            x_part(3, 2, xs + 544);
            __syncthreads();
            t_part(1, 0, xs);
            t_part(2, 1, xs + 272);
            t_part(3, 2, xs + 544);
            __syncthreads();
            x_part(2, 0, xs);
            x_part(3, 1, xs + 272);
            __syncthreads();
            t_part(2, 0, xs);
            t_part(3, 1, xs + 272);
            __syncthreads();
            x_part(3, 0, xs);
            __syncthreads();
            t_part(3, 0, xs);   // A is no longer read: P may use its space
            if (!strong && !is_k) {   // P (lanes 64..127), lower with the diagonal -> AM
                float vv[32];
                tmem_ld32_sync(D1 + lane_base + 32 * hc, vv);
                const int r = r_el;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int i = 32 * hc + e;
                    am[r * LDA + i] = i <= r ? vv[e] : 0.f;
                }
            }
            __syncthreads();
            // T diag(beta) -> TMEM (hi | lo), MMA2's A operand (lanes 0..63)
            if (is_k) {
                float th[32], tl[32];
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    split_tf32(tt[row * LDA + 32 * hc + e] * s_beta[32 * hc + e], th[e], tl[e]);
                tmem_st32_sync(A2 + lane_base + 32 * hc, th);
                tmem_st32_sync(A2 + 64 + lane_base + 32 * hc, tl);
            }
            __syncthreads();   // T is read: V^T may take its space
        }
        // ---- V^T (hi | lo) over K-m (MMA2's B operand); the P record from AM
        {
            const float* vs = reinterpret_cast<const float*>(sm + Sm::VS);
            const uint32_t vt_lo = 2u * DV * 128u;
            for (int idx = tid; idx < 64 * (DV / 4); idx += 256) {
                const int r = idx & 63, c4 = (idx >> 6) * 4;
                const float4 x4 = *reinterpret_cast<const float4*>(vs + r * LDV + c4);
                const float xv[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float hi, lo;
                    split_tf32(xv[e], hi, lo);
                    const uint32_t off = (uint32_t)(r >> 5) * (DV * 128u) + sw128_offset(c4 + e, (r & 31) * 4);
                    *reinterpret_cast<float*>(sm + Sm::KB + off) = hi;
                    *reinterpret_cast<float*>(sm + Sm::KB + vt_lo + off) = lo;
                }
            }
            if (!strong) {
                // record tiles: [half t][row][32 floats], 16-byte chunks swizzled by row
                for (int idx = tid; idx < 1024; idx += 256) {
                    const int th = idx >> 9, rr = (idx >> 3) & 63, lc = (idx & 7) ^ (rr & 7);
                    const float* src = am + rr * LDA + 32 * th + 4 * lc;
                    *reinterpret_cast<float4*>(rec + R::P + (size_t)idx * 4) = make_float4(src[0], src[1], src[2], src[3]);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- MMA2: W = T diag(beta) K~, U0 = T diag(beta) V (split tf32, K = 64 tokens)
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idw = instr_desc(kFmtTF32, 128, DK);
            constexpr uint32_t idu = instr_desc(kFmtTF32, 128, DV);
            const uint32_t kt = smem_u32(sm + Sm::KTT), vt = smem_u32(sm + Sm::KB);
#pragma unroll
            for (int pass = 0; pass < 3; ++pass) {
                const uint32_t acol = pass == 1 ? 64 : 0;
                const uint32_t kofs = pass == 0 ? 2u * DK * 128u : 0, vofs = pass == 0 ? 2u * DV * 128u : 0;
#pragma unroll
                for (int t = 0; t < 2; ++t)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint32_t a = A2 + acol + t * 32 + ks * 8;
                        const bool acc = (pass | t | ks) != 0;
                        mma_tf32_ts(D2, a, smem_desc(kt + kofs + t * (DK * 128u) + ks * 32, 16, 1024, kLayoutSW128),
                                    idw, acc);
                        mma_tf32_ts(D2 + DK, a, smem_desc(vt + vofs + t * (DV * 128u) + ks * 32, 16, 1024, kLayoutSW128),
                                    idu, acc);
                    }
            }
            mma_commit(&bar_mma);
        }
        mma_pending = 1;
        if (!wait_mma()) { aborted = true; break; }
        if (has_next) prefetch_kq(w + gridDim.x);   // the operand tiles are dead
        // ---- W, U0 (lanes 0..63) -> staging over G, AM, VS, then coalesced
        //      stores; then the next item's log-decay tile into G
        if (is_k) {
            float* ws = reinterpret_cast<float*>(sm + Sm::WS);
            float* us = reinterpret_cast<float*>(sm + Sm::US);
#pragma unroll
            for (int cb = 0; cb < DK / 2; cb += 32) {
                float vv[32];
                tmem_ld32_sync(D2 + lane_base + hc * (DK / 2) + cb, vv);
                float* dst = ws + row * LDK + hc * (DK / 2) + cb;
#pragma unroll
                for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(dst + e) = make_float4(vv[e], vv[e + 1], vv[e + 2], vv[e + 3]);
            }
#pragma unroll
            for (int cb = 0; cb < DV / 2; cb += 32) {
                float vv[32];
                tmem_ld32_sync(D2 + DK + lane_base + hc * (DV / 2) + cb, vv);
                float* dst = us + row * LDV + hc * (DV / 2) + cb;
#pragma unroll
                for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(dst + e) = make_float4(vv[e], vv[e + 1], vv[e + 2], vv[e + 3]);
            }
        }
        __syncthreads();
        {
            const float* ws = reinterpret_cast<const float*>(sm + Sm::WS);
            const float* us = reinterpret_cast<const float*>(sm + Sm::US);
            for (int idx = tid; idx < 64 * (DK / 4); idx += 256) {
                const int r = idx / (DK / 4), c4 = (idx - r * (DK / 4)) * 4;
                *reinterpret_cast<float4*>(rec + R::WQ + (size_t)r * DK + c4) = *reinterpret_cast<const float4*>(ws + r * LDK + c4);
            }
            // U0 as 32-column slices [DV/32][row][32 floats], 16-byte chunks swizzled by row
            for (int idx = tid; idx < 64 * (DV / 4); idx += 256) {
                const int jt = idx >> 9, rr = (idx >> 3) & 63, lc = (idx & 7) ^ (rr & 7);
                *reinterpret_cast<float4*>(rec + R::U0 + (size_t)idx * 4) =
                    *reinterpret_cast<const float4*>(us + rr * LDV + 32 * jt + 4 * lc);
            }
        }
        tc_fence_before();
        __syncthreads();   // TMEM, g, A / T and the staging are reused by the next item
        tc_fence_after();
        if (has_next) prefetch_la(w + gridDim.x);
    }

    if (aborted) {
        if (tid == 0) {
            flag_error(hdr, kStatusTimeout);
            if (mma_pending) (void)mbar_wait_cycles(&bar_mma, mma_phase, kWaitCycles);
        }
        cp_async_wait<0>();   // a prefetch may still be landing in shared memory
        __syncthreads();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int DK, int DV, int GATE>
cudaError_t launch_intra_f32_tc_t(const ChunkArgs& a) {
    ChunkMap map{a.cu_seqlens, a.chunk_offsets, a.num_seqs, a.T, a.fixed_chunks_per_seq};
    auto kern = intra_chunk_f32_tc_kernel<DK, DV, GATE>;
    const int smem = (int)F32K1Smem<DK, DV>::END + 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const size_t items = a.max_chunks * (size_t)a.H;
    const unsigned grid = (unsigned)(items < (size_t)sms ? items : (size_t)sms);
    kern<<<grid, 256, smem, a.stream>>>(static_cast<const float*>(a.q), static_cast<const float*>(a.k),
                                        static_cast<const float*>(a.v), a.log_alpha, a.beta, map,
                                        static_cast<WsHeader*>(a.ws_header), static_cast<float*>(a.records), a.H,
                                        a.max_chunks);
    return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_intra_f32_tc_g(const ChunkArgs& a) {
    if (a.gate == kGateChannel) return launch_intra_f32_tc_t<DK, DV, kGateChannel>(a);
    if (a.gate == kGateHead) return launch_intra_f32_tc_t<DK, DV, kGateHead>(a);
    return launch_intra_f32_tc_t<DK, DV, kGateNone>(a);
}

}  // namespace

cudaError_t launch_chunk_intra_f32_tc(const ChunkArgs& a) {
    if (a.max_chunks == 0 || a.H == 0) return cudaSuccess;
    if (a.dk == 128 && a.dv == 128) return launch_intra_f32_tc_g<128, 128>(a);
    if (a.dk == 128 && a.dv == 64) return launch_intra_f32_tc_g<128, 64>(a);
    if (a.dk == 64 && a.dv == 128) return launch_intra_f32_tc_g<64, 128>(a);
    if (a.dk == 64 && a.dv == 64) return launch_intra_f32_tc_g<64, 64>(a);
    return cudaErrorInvalidValue;
}

}  // namespace kda
