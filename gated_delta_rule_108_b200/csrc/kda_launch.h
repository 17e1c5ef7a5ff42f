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
    void* records;                // per (head, chunk) intermediates
    size_t max_chunks;            // chunks per head the records can hold
    int fixed_chunks_per_seq;     // ceil(T / 64) for fixed length
    cudaStream_t stream;
};

// Bytes of per-(head, chunk) intermediates: fp32 CUDA-core path / bf16 tensor-core path.
size_t simt_record_bytes(int dk, int dv);
size_t tc_record_bytes(int dk, int dv);

// Sets the calling thread's kda_last_error() message and returns `status`
// (status is a kda_status value).
int set_error(int status, const char* fmt, ...);

cudaError_t launch_decode(const DecodeArgs& a);
cudaError_t launch_chunk_prep(const ChunkArgs& a);     // K0: status reset + varlen chunk table
cudaError_t launch_chunk_intra(const ChunkArgs& a);    // K1: all chunks in parallel
cudaError_t launch_chunk_inter(const ChunkArgs& a);    // K2: serial over each sequence's chunks
cudaError_t launch_chunk_intra_tc(const ChunkArgs& a); // bf16 inputs: tensor-core K1
cudaError_t launch_chunk_inter_tc(const ChunkArgs& a); // bf16 inputs: tensor-core K2

}  // namespace kda
