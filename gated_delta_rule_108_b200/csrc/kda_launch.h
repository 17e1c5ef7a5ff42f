// kda_launch.h -- internal launcher interface between the C ABI (kda_api.cu)
// and the kernel files.  Not installed; the public ABI is include/kda.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kda {

struct DecodeArgs {
    const void* q; const void* k; const void* v;
    const float* log_alpha; const float* beta;
    float* state; void* o;
    int B, H, dk, dv;
    int gate;                     // kGateChannel: log_alpha [B,H,dk]; kGateHead: [B,H]; kGateNone: unused
    bool bf16;
    float scale;
    cudaStream_t stream;
};

// Everything the chunkwise kernels need for one kda_chunk_fwd call.
struct ChunkArgs {
    const void* q; const void* k; const void* v;
    const float* log_alpha; const float* beta;
    const float* initial_state;   // nullable
    const int32_t* cu_seqlens;    // nullable
    void* o; float* final_state;  // final_state nullable
    int B, T, H, dk, dv, num_seqs;
    int gate;                     // kGateChannel: log_alpha [.., H, dk]; kGateHead: [.., H]; kGateNone: unused
    bool bf16;
    float scale;
    // workspace carve-up (computed by the ABI layer)
    void* ws_header;              // WsHeader
    int32_t* chunk_offsets;       // [N+1], varlen only
    int32_t* seq_order;           // [N] packed sequences longest first (bf16 forward, N > 1), else null
    void* records;                // per (head, chunk) intermediates
    size_t max_chunks;            // chunks per head the records can hold
    int fixed_chunks_per_seq;     // ceil(T / 64) for fixed length
    cudaStream_t stream;
    // backward pass only (all null in the forward)
    float* tmat;                  // [H][max_chunks][64][64]: the fp32 K1 also writes T = (I + A)^{-1}
    void* bwd_tiles;              // bf16: [H][max_chunks] fp16 T, K~, V tiles and fp32 M from the tensor-core K1
    int* bwd_flags;               // bf16: [H][max_chunks] 1 where the chunk took the strong-decay path
    float* states;                // [H][max_chunks][dk][dv]: K2 also writes the state entering each chunk
    const void* d_o;              // [.., H, dv], input dtype
    const float* d_final_state;   // [N, H, dk, dv], nullable (zeros)
    void* dq; void* dk_out; void* dv_out;   // input dtype
    float* dlog_alpha; float* dbeta;
    float* d_initial_state;       // [N, H, dk, dv], nullable (not written)
    float* dS_end;                // [H][max_chunks][dk][dv]: dL/d(state leaving each chunk)
    float* dU;                    // [H][max_chunks][64][dv]: dL/dU of each chunk
    float* scratch;               // per-CTA fp32 scratch of the per-chunk gradient kernel
    float* vside;                 // bf16: [H][max_chunks] VSide blocks from the value-side kernel (else null)
    int bwd_ctas;                 // CTAs of that kernel (its scratch holds this many)
    // test hook (kda_debug_drop_copy): the tensor-core intra-chunk kernel leaves
    // out one copy and caps its waits at wait_cap cycles (0: the default cap)
    int debug_drop_copy;
    long long wait_cap;
};

// Bytes of per-(head, chunk) intermediates: fp32 CUDA-core path / bf16 tensor-core path.
size_t simt_record_bytes(int dk, int dv);
size_t tc_record_bytes(int dk, int dv);
size_t bwd_tiles_bytes(int dk, int dv);   // the tensor-core K1's backward-mode block per (head, chunk)

// Sets the calling thread's kda_last_error() message and returns `status`
// (status is a kda_status value).
int set_error(int status, const char* fmt, ...);

cudaError_t launch_decode(const DecodeArgs& a);
cudaError_t launch_chunk_prep(const ChunkArgs& a);     // K0: status reset + varlen chunk table
cudaError_t launch_chunk_intra(const ChunkArgs& a);    // K1: all chunks in parallel
cudaError_t launch_chunk_inter(const ChunkArgs& a);    // K2: serial over each sequence's chunks
cudaError_t launch_chunk_intra_tc(const ChunkArgs& a); // bf16 inputs: tensor-core K1
cudaError_t launch_chunk_intra_f32_tc(const ChunkArgs& a); // fp32 inputs, forward: tensor-core K1 (split tf32)
cudaError_t launch_chunk_intra_fwd_tc(const ChunkArgs& a); // its forward-only form, two CTAs per SM
cudaError_t launch_chunk_inter_tc(const ChunkArgs& a); // bf16 inputs: tensor-core K2
cudaError_t launch_chunk_inter_fwd_tc(const ChunkArgs& a); // its forward-only form, slice width per call
cudaError_t launch_chunk_inter_f32_tc(const ChunkArgs& a); // fp32 inputs, forward: tensor-core K2 (split tf32)
cudaError_t launch_chunk_fused_tc(const ChunkArgs& a);     // bf16 forward in one pass, one CTA per (sequence, head)
cudaError_t launch_chunk_seq_order(const ChunkArgs& a);    // packed sequences longest first into a.seq_order
cudaError_t launch_chunk_bwd_inter(const ChunkArgs& a);  // backward: serial over chunks, reversed
cudaError_t launch_chunk_bwd_inter_tc(const ChunkArgs& a); // the same on the tensor cores (bf16 inputs)
cudaError_t launch_chunk_bwd_vside_tc(const ChunkArgs& a); // backward products over the value dim (bf16 inputs)
cudaError_t launch_chunk_bwd_tchain_tc(const ChunkArgs& a); // backward products through T, W, U0 (bf16 inputs)
cudaError_t launch_chunk_bwd_split_tc(const ChunkArgs& a);  // backward split-factor products and gradients (bf16)
cudaError_t launch_chunk_bwd_intra(const ChunkArgs& a);  // backward: all chunks in parallel
size_t bwd_scratch_bytes_per_cta(int dk, int dv);
constexpr int kBwdMaxCtas = 512;   // scratch is sized for at most this many CTAs

}  // namespace kda
