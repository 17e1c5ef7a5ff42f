// kda_tc_common.cuh -- definitions shared by the tensor-core kernel files of
// libkda_b200 (sm_100a): the fp16 record of one (head, chunk) that the
// intra-chunk kernels write and the inter-chunk kernels read, constants, the
// exact A / P of strong-decay chunks, and the TMA descriptor helpers.
#pragma once

#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kda_common.cuh"
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


// Backward mode of the intra-chunk kernel, per (head, chunk): T = (I + A)^{-1},
// K~ = k e^{g} and V as fp16 128-byte-swizzled tiles of 64 rows (token) by 64
// columns, the operands of the backward's T-chain products.
template <int DK, int DV>
struct BwdTiles {
    static constexpr uint32_t T = 0;
    static constexpr uint32_t KT = T + 8192;
    static constexpr uint32_t V = KT + (DK / 64) * 8192;
    static constexpr uint32_t TILE_BYTES = V + (DV / 64) * 8192;   // the fp16 tiles
    static constexpr uint32_t M = TILE_BYTES;                       // fp32 M = K_l K_r^T [64][64], strictly lower
    static constexpr uint32_t BYTES = M + 64 * 64 * 4;
};

constexpr float kMaxSplitExponent = 60.f;   // e^60 ~ 1e26: far inside the fp32 range
// The intra-chunk kernel keeps the cumulative log-decay in base 2 (g log2(e)),
// so each factor e^{x} is one hardware 2^{x}.
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kMaxSplitExponent2 = kMaxSplitExponent * kLog2e;
constexpr int kCopyThread = 32;     // the intra-chunk kernel's TMA / bulk-copy thread (warp 1)
constexpr int kTileThread = 128;    // its backward-mode tile stores (warp 4, idle in the diagonal solve)

// Exact A and P of one chunk, used when its decay is too strong for the split
// factors (g in base 2, read through gat(token, channel)): A_ri = beta_r sum_c
// k_rc k_ic e^{g_rc - g_ic} (i < r) into am [64][lda] (zero on and above the
// diagonal) and P_ri = sum_c q_rc k_ic e^{g_rc - g_ic} (i <= r) as fp16 into the
// record's P tile.  Every exponent is <= 0.  One warp per (r, i) pair, lanes
// over channels; k and q are the bf16 tiles as loaded.
template <int DK, class GAt>
__device__ __forceinline__ void exact_a_p(GAt gat, const unsigned char* ks, const unsigned char* qs,
                                          const float* s_beta, int L, float* am, unsigned char* prec,
                                          int lda = 68)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int pr = warp; pr < 64 * 64; pr += 8) {
        const int r = pr >> 6, i = pr & 63;
        float sa = 0.f, sp = 0.f;
        if (i <= r && r < L) {
#pragma unroll
            for (int c0 = 0; c0 < DK; c0 += 32) {
                const int c = c0 + lane;
                const uint32_t hr = (c >> 6) * 8192u + sw128_offset(r, (c & 63) * 2);
                const uint32_t hi = (c >> 6) * 8192u + sw128_offset(i, (c & 63) * 2);
                const float w = ex2_approx(gat(r, c) - gat(i, c));
                const float ki = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(ks + hi));
                const float kr = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(ks + hr));
                const float qr = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(qs + hr));
                sa += kr * ki * w;
                sp += qr * ki * w;
            }
#pragma unroll
            for (int off = 16; off; off >>= 1) {
                sa += __shfl_xor_sync(0xffffffffu, sa, off);
                sp += __shfl_xor_sync(0xffffffffu, sp, off);
            }
        }
        if (lane == 0) {
            am[r * lda + i] = (i < r) ? s_beta[r] * sa : 0.f;
            *reinterpret_cast<__half*>(prec + sw128_offset(r, i * 2)) = __float2half_rn(sp);
        }
    }
}

// ------------------------------------------------------------- host -----
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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
inline bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, int d, int H,
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


}  // namespace
}  // namespace kda
