// kda_common.cuh -- shared device/host helpers of libkda_b200 (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

constexpr int kChunk = 64;          // tokens per chunk in the chunkwise form
constexpr int kHeaderBytes = 256;   // workspace header (status word, counts)

// Device status codes written into the workspace header (same values as
// kda_status in include/kda.h).
constexpr int kStatusOk = 0;
constexpr int kStatusInternal = 3;   // reported as KDA_ERR_CUDA
constexpr int kStatusTimeout = 4;
constexpr int kStatusBadSeqlens = 6;
constexpr int kStatusRange = 7;

// Decay gate kinds (same values as kda_gate in include/kda.h): one log-decay
// per key channel (KDA), one per head (Gated DeltaNet), or none (DeltaNet).
constexpr int kGateChannel = 0;
constexpr int kGateHead = 1;
constexpr int kGateNone = 2;

// Workspace header, at offset 0 of the caller's workspace.
struct WsHeader {
    int status;       // argument check of the last call (0 = ok): kernels skip work if set
    int num_chunks;   // chunks per head in this call
    int runtime_err;  // first error a kernel hit while working (0 = none), e.g. a timeout
    int next_pair;    // fused forward: next (sequence, head) pair to claim
    int reserved[60];
};
static_assert(sizeof(WsHeader) == kHeaderBytes, "header size");

// fp32 record of one (head, chunk), row-major: W [64][DK] | U0 [64][DV] |
// Q~ [64][DK] | K^ [64][DK] | P [64][64] | gamma [DK].  Rows past the chunk's
// tokens are zero.  Written by the CUDA-core intra-chunk kernel (fp32 inputs);
// read by the CUDA-core inter-chunk kernel and the fp32 backward kernels.
template <int DK, int DV>
struct F32Rec {
    static constexpr size_t W = 0;
    static constexpr size_t U0 = W + kChunk * DK;
    static constexpr size_t QT = U0 + kChunk * DV;
    static constexpr size_t KH = QT + kChunk * DK;
    static constexpr size_t P = KH + kChunk * DK;
    static constexpr size_t GC = P + kChunk * kChunk;
    static constexpr size_t FLOATS = (GC + DK + 63) / 64 * 64;   // 256-byte multiple
};

// The same quantities for the fp32 tensor-core kernels, laid out for them:
//   WQ  [128][DK]  rows 0..63 W, 64..127 Q~ (row-major; one thread loads a row)
//   KHT [DK][64]   K^ transposed (row = key channel, one thread loads a row)
//   P   [2][64][32] the two 32-token halves of P, each row's 16-byte chunks
//                  XOR-swizzled by (row mod 8) (the 128-byte swizzle of an MMA tile)
//   U0  [DV/32][64][32] 32-column slices of U0, swizzled the same way
//   GC  [DK]
// Rows past the chunk's tokens are zero.  Same size as F32Rec.
template <int DK, int DV>
struct F32TcRec {
    static constexpr size_t WQ = 0;
    static constexpr size_t KHT = WQ + 2 * kChunk * DK;
    static constexpr size_t P = KHT + DK * kChunk;
    static constexpr size_t U0 = P + kChunk * kChunk;
    static constexpr size_t GC = U0 + kChunk * DV;
    static constexpr size_t FLOATS = (GC + DK + 63) / 64 * 64;
    static_assert(FLOATS == F32Rec<DK, DV>::FLOATS, "the workspace is sized by F32Rec");
};

// Backward, per (head, chunk), fp32: the products over the value dimension,
// dQ~ = D S^T, dW = -dU S^T, dK^ = U dS'^T [64][DK] each, dP = D U^T [64][64]
// (lower with the diagonal), dgamma [DK].  Written by the tensor-core
// value-side kernel (bf16 inputs), read by the per-chunk gradient kernel.
// Then the T-chain products (tensor-core T-chain kernel): dK~ = beta T^T dW
// [64][DK], dA = -T^T dT T^T [64][64] (strictly lower) and the parts of dbeta
// that come through W and U0 [64].
template <int DK>
struct VSide {
    static constexpr size_t DQT = 0;
    static constexpr size_t DW = DQT + kChunk * DK;
    static constexpr size_t DKH = DW + kChunk * DK;
    static constexpr size_t DP = DKH + kChunk * DK;
    static constexpr size_t DGAM = DP + kChunk * kChunk;
    static constexpr size_t DKT = DGAM + DK;
    static constexpr size_t DA = DKT + kChunk * DK;
    static constexpr size_t DBP = DA + kChunk * kChunk;
    static constexpr size_t FLOATS = (DBP + kChunk + 63) / 64 * 64;
};

// Element loads/stores for the two input dtypes.
template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Where the tokens of one chunk live.  Sequences are either B rows of T
// tokens (fixed) or packed by cu_seqlens (varlen); chunks never cross a
// sequence boundary and the last chunk of a sequence may be short.
struct ChunkMap {
    const int32_t* cu_seqlens;     // varlen: [N+1]; nullptr for fixed length
    const int32_t* chunk_offsets;  // varlen: [N+1] first chunk of each sequence
    int num_seqs;                  // N
    int T;                         // fixed: tokens per sequence; varlen: total
    int chunks_per_seq;            // fixed: ceil(T / 64)

    __device__ __forceinline__ int seq_first_chunk(int s) const {
        return cu_seqlens ? chunk_offsets[s] : s * chunks_per_seq;
    }
    __device__ __forceinline__ int seq_num_chunks(int s) const {
        return cu_seqlens ? chunk_offsets[s + 1] - chunk_offsets[s] : chunks_per_seq;
    }
    __device__ __forceinline__ int seq_token_begin(int s) const {
        return cu_seqlens ? cu_seqlens[s] : s * T;
    }
    __device__ __forceinline__ int seq_token_end(int s) const {
        return cu_seqlens ? cu_seqlens[s + 1] : (s + 1) * T;
    }
    // Global chunk index -> (sequence, first token, length).
    __device__ __forceinline__ void locate(int c, int& s, int& tok0, int& len) const {
        if (!cu_seqlens) {
            s = c / chunks_per_seq;
            const int j = c - s * chunks_per_seq;
            tok0 = s * T + j * kChunk;
            len = min(kChunk, T - j * kChunk);
            return;
        }
        // largest s with chunk_offsets[s] <= c (skips empty sequences)
        int lo = 0, hi = num_seqs - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (chunk_offsets[mid] <= c) lo = mid; else hi = mid - 1;
        }
        s = lo;
        tok0 = cu_seqlens[s] + (c - chunk_offsets[s]) * kChunk;
        len = min(kChunk, cu_seqlens[s + 1] - tok0);
    }
};

}  // namespace kda
