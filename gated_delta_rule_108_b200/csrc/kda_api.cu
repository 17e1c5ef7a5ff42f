// kda_api.cu -- the C ABI of libkda_b200 (declared in include/kda.h).
//
// Validates arguments, carves the caller's workspace, and enqueues the
// kernels on the caller's stream.  Nothing here allocates device memory or
// synchronises, except kda_workspace_status.
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#include "../../include/kda.h"
#include "kda_common.cuh"
#include "kda_launch.h"

namespace {

thread_local std::string g_last_error;
thread_local long long g_debug_drop_cap = 0;   // armed by kda_debug_drop_copy (one call)
constexpr int kMaxStageEvents = 7;
thread_local cudaEvent_t g_stage_events[kMaxStageEvents] = {};
thread_local int g_stage_event_count = 0;   // 0: off

cudaError_t mark_stage(int i, cudaStream_t s) {
    return i < g_stage_event_count ? cudaEventRecord(g_stage_events[i], s) : cudaSuccess;
}

kda_status fail(kda_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

kda_status ok() {
    g_last_error.clear();
    return KDA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool supported_dim(int d) { return d == 64 || d == 128; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace carve-up: [header 256 B][chunk_offsets (N+1) int32][sequence order
// N int32 (packed inputs: longest first)][records], each part 256-byte aligned.
struct WsLayout {
    size_t offsets_off, order_off, records_off, total;
    size_t max_chunks;
    int chunks_per_seq;
};

bool ws_layout(int B, int T, int H, int dk, int dv, int num_seqs, bool varlen, kda_dtype dtype,
               WsLayout& L) {
    if (B < 0 || T < 0 || H <= 0 || !supported_dim(dk) || !supported_dim(dv)) return false;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return false;
    const int N = varlen ? num_seqs : B;
    if (N < 0 || (varlen && B != 1)) return false;
    L.chunks_per_seq = (T + kda::kChunk - 1) / kda::kChunk;
    if (varlen) {
        // each sequence of length l holds ceil(l/64) <= (l + 63)/64 chunks
        L.max_chunks = ((size_t)T + 63u * (size_t)N) / kda::kChunk;
    } else {
        L.max_chunks = (size_t)B * L.chunks_per_seq;
    }
    // bf16 inputs: fp16 records; fp32 inputs: fp32 records, of one size for
    // the split-tf32 tensor-core forward and for the CUDA-core kernels of the
    // backward's recomputation.
    const size_t rec = dtype == KDA_BF16 ? kda::tc_record_bytes(dk, dv) : kda::simt_record_bytes(dk, dv);
    L.offsets_off = kda::kHeaderBytes;
    L.order_off = round_up(L.offsets_off + sizeof(int32_t) * ((size_t)N + 1), 256);
    L.records_off = round_up(L.order_off + sizeof(int32_t) * (size_t)N, 256);
    L.total = L.records_off + rec * (size_t)H * L.max_chunks;
    return true;
}

// Backward workspace: [header][chunk_offsets][the forward's records][bf16
// inputs: the tensor-core products, fp16 T / K~ / V tiles; fp32 inputs: T]
// [chunk-start states][dS at chunk ends][dU][per-CTA scratch], each 256-byte
// aligned.
struct BwdLayout {
    WsLayout base;   // header, offsets, the forward's records for this dtype
    size_t vside_off;// bf16: the tensor-core products per (head, chunk) (0 for fp32)
    size_t tiles_off;// bf16: fp16 T, K~, V tiles, fp32 M per (head, chunk) (0 for fp32)
    size_t flags_off;// bf16: strong-decay flag per (head, chunk) (0 for fp32)
    size_t tmat_off, states_off, dS_off, dU_off, scratch_off, total;
    int ctas;        // CTAs the scratch holds
};

bool bwd_layout(int B, int T, int H, int dk, int dv, int num_seqs, bool varlen, kda_dtype dtype,
                BwdLayout& L) {
    if (!ws_layout(B, T, H, dk, dv, num_seqs, varlen, dtype, L.base)) return false;
    const size_t units = (size_t)H * L.base.max_chunks;   // (head, chunk) pairs
    size_t off = round_up(L.base.total, 256);
    L.vside_off = 0;
    L.tiles_off = 0;
    L.flags_off = 0;
    L.tmat_off = 0;
    if (dtype == KDA_BF16) {
        L.vside_off = off;
        const size_t vs_floats = dk == 128 ? kda::VSide<128>::FLOATS : kda::VSide<64>::FLOATS;
        off = round_up(off + sizeof(float) * vs_floats * units, 256);
        L.tiles_off = off;
        off = round_up(off + kda::bwd_tiles_bytes(dk, dv) * units, 256);   // fp16 T, K~, V tiles, fp32 M
        L.flags_off = off;
        off = round_up(off + sizeof(int) * units, 256);
    } else {
        L.tmat_off = off;
        off = round_up(off + sizeof(float) * kda::kChunk * kda::kChunk * units, 256);
    }
    const size_t after_t = off;
    L.states_off = after_t;
    L.dS_off = round_up(L.states_off + sizeof(float) * (size_t)dk * dv * units, 256);
    L.dU_off = round_up(L.dS_off + sizeof(float) * (size_t)dk * dv * units, 256);
    L.scratch_off = round_up(L.dU_off + sizeof(float) * kda::kChunk * (size_t)dv * units, 256);
    L.ctas = (int)(units < (size_t)kda::kBwdMaxCtas ? units : (size_t)kda::kBwdMaxCtas);
    L.total = L.scratch_off + kda::bwd_scratch_bytes_per_cta(dk, dv) * (size_t)L.ctas;
    return true;
}

// Which form of the bf16 chunk forward runs.  The two-kernel split form (all
// chunks in parallel at two CTAs per SM, records through the workspace, then
// the chunk-to-chunk recurrence) is the faster one on B200 at every workload
// measured, so it runs whenever the workspace holds the records.  The fused
// single pass (one CTA per (sequence, head) pair, each chunk's intermediates
// kept on chip) needs only the header, the chunk table and the pair order, and
// runs when the workspace is smaller than that.  KDA_CHUNK_PATH = "fused" /
// "split" forces one (tests, measurements); "auto" or unset decides.
int chunk_path_override() {
    const char* e = getenv("KDA_CHUNK_PATH");
    if (!e || !*e || strcmp(e, "auto") == 0) return 0;
    if (strcmp(e, "fused") == 0) return 1;
    if (strcmp(e, "split") == 0) return 2;
    return 0;
}

// Workspace bytes of the fused single pass: the header, the chunk table and
// the sequence order (everything before the records).
size_t fused_ws_bytes(int N, bool varlen, const WsLayout& L) {
    (void)N; (void)varlen;
    return L.records_off;
}

// fused (1) or split (0) for a workspace of ws_bytes (SIZE_MAX: as large as needed)
int chunk_fwd_fused(int N, bool varlen, kda_dtype dtype, const WsLayout& L, size_t ws_bytes) {
    if (dtype != KDA_BF16) return 0;
    const size_t fused_need = fused_ws_bytes(N, varlen, L);
    const int ov = chunk_path_override();
    if (ov == 1) return ws_bytes >= fused_need ? 1 : 0;
    if (ov == 2) return 0;
    return (ws_bytes < L.total && ws_bytes >= fused_need) ? 1 : 0;
}

}  // namespace

namespace kda {
int set_error(int status, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return status;
}
}  // namespace kda

extern "C" {

size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs, int varlen,
                                    kda_dtype dtype) {
    WsLayout L;
    if (!ws_layout(B, T, H, dk, dv, num_seqs, varlen != 0, dtype, L)) return 0;
    return L.total;
}

// save: the workspace has the backward's layout, and the forward kernels run in
// backward mode, so that it also holds what kda_chunk_bwd would recompute.
static kda_status chunk_fwd_impl(const void* q, const void* k, const void* v, const float* log_alpha,
                                 const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                                 int B, int T, int H, int dk, int dv, int num_seqs, kda_dtype dtype,
                                 kda_gate gate, void* o, float* final_state, void* workspace,
                                 size_t workspace_bytes, void* stream, bool save = false) {
    if (dtype != KDA_F32 && dtype != KDA_BF16) return fail(KDA_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (gate != KDA_GATE_CHANNEL && gate != KDA_GATE_HEAD && gate != KDA_GATE_NONE)
        return fail(KDA_ERR_INVALID_ARG, "unknown gate kind %d", (int)gate);
    if (B < 0 || T < 0 || H <= 0) return fail(KDA_ERR_INVALID_ARG, "bad sizes B=%d T=%d H=%d", B, T, H);
    if (dk <= 0 || dv <= 0) return fail(KDA_ERR_INVALID_ARG, "bad head sizes dk=%d dv=%d", dk, dv);
    if (!supported_dim(dk) || !supported_dim(dv))
        return fail(KDA_ERR_UNSUPPORTED, "head sizes dk=%d dv=%d not in {64, 128}", dk, dv);
    const bool varlen = cu_seqlens != nullptr;
    if (varlen && B != 1) return fail(KDA_ERR_INVALID_ARG, "cu_seqlens requires B == 1 (got B=%d)", B);
    if (varlen && num_seqs < 0) return fail(KDA_ERR_INVALID_ARG, "num_seqs=%d < 0", num_seqs);
    const int N = varlen ? num_seqs : B;
    const size_t tokens = varlen ? (size_t)T : (size_t)B * T;
    if (tokens * (size_t)H * (size_t)(dk > dv ? dk : dv) >= (size_t)1 << 31)
        return fail(KDA_ERR_UNSUPPORTED, "B*T*H*d = %zu elements exceeds 2^31", tokens * H * (dk > dv ? dk : dv));
    if (tokens > 0) {
        if (!q || !k || !v || !beta || !o || (gate != KDA_GATE_NONE && !log_alpha))
            return fail(KDA_ERR_INVALID_ARG, "null input/output pointer");
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
            (gate == KDA_GATE_CHANNEL && !aligned16(log_alpha)))
            return fail(KDA_ERR_INVALID_ARG, "q/k/v/log_alpha/o must be 16-byte aligned");
    }
    if (initial_state && !aligned16(initial_state)) return fail(KDA_ERR_INVALID_ARG, "initial_state misaligned");
    if (final_state && !aligned16(final_state)) return fail(KDA_ERR_INVALID_ARG, "final_state misaligned");
    if (initial_state && final_state && initial_state != final_state) {
        const char* a0 = (const char*)initial_state;
        const char* b0 = (const char*)final_state;
        const size_t bytes = (size_t)N * H * dk * dv * sizeof(float);
        if (a0 < b0 + bytes && b0 < a0 + bytes)
            return fail(KDA_ERR_INVALID_ARG, "initial_state and final_state overlap without being equal");
    }
    BwdLayout LB;
    if (!bwd_layout(B, T, H, dk, dv, num_seqs, varlen, dtype, LB))
        return fail(KDA_ERR_INVALID_ARG, "invalid sizes for the workspace layout");
    const WsLayout& L = LB.base;   // the backward layout starts with the forward's
    const size_t need = save ? LB.total : L.total;
    if (!workspace) return fail(KDA_ERR_WORKSPACE, "workspace is null (need %zu bytes)", need);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(KDA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    // a training forward (save) runs the two-kernel form in backward mode
    const int fused = save ? 0 : chunk_fwd_fused(N, varlen, dtype, L, workspace_bytes);
    if (workspace_bytes < need && !fused)
        return fail(KDA_ERR_WORKSPACE, "workspace has %zu bytes, need %zu%s", workspace_bytes, need,
                    dtype == KDA_BF16 && !save ? " (or the fused pass's kda_chunk_fwd_fused_workspace_size)" : "");

    kda::ChunkArgs a{};
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.initial_state = initial_state; a.cu_seqlens = cu_seqlens;
    a.o = o; a.final_state = final_state;
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv; a.num_seqs = N;
    a.gate = (int)gate;
    a.bf16 = dtype == KDA_BF16;
    a.scale = 1.0f / sqrtf((float)dk);
    a.ws_header = workspace;
    a.chunk_offsets = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + L.offsets_off);
    a.seq_order = (a.bf16 && varlen && N > 1 && !save) ? reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + L.order_off)
                                             : nullptr;
    a.records = static_cast<char*>(workspace) + L.records_off;
    a.max_chunks = L.max_chunks;
    a.fixed_chunks_per_seq = L.chunks_per_seq;
    a.stream = static_cast<cudaStream_t>(stream);
    if (save) {   // backward mode: T (and for bf16 the K~, V tiles, M, strong-decay flags), chunk-start states
        char* ws = static_cast<char*>(workspace);
        a.tmat = a.bf16 ? nullptr : reinterpret_cast<float*>(ws + LB.tmat_off);
        a.bwd_tiles = a.bf16 ? static_cast<void*>(ws + LB.tiles_off) : nullptr;
        a.bwd_flags = a.bf16 ? reinterpret_cast<int*>(ws + LB.flags_off) : nullptr;
        a.states = reinterpret_cast<float*>(ws + LB.states_off);
    }
    if (g_debug_drop_cap > 0 && a.bf16 && gate == KDA_GATE_CHANNEL) {   // one-shot test hook
        a.debug_drop_copy = 1;
        a.wait_cap = g_debug_drop_cap;
        g_debug_drop_cap = 0;
    }

    cudaError_t e = mark_stage(0, a.stream);
    if (e == cudaSuccess) e = kda::launch_chunk_prep(a);
    if (e == cudaSuccess && a.bf16 && a.seq_order) e = kda::launch_chunk_seq_order(a);   // longest first
    if (e == cudaSuccess) e = mark_stage(1, a.stream);
    if (fused) {   // one pass; the inter-chunk stage is empty
        if (e == cudaSuccess) e = kda::launch_chunk_fused_tc(a);
        if (e == cudaSuccess) e = mark_stage(2, a.stream);
    } else {
        // fp32: the split-tf32 tensor-core K1, or in backward mode (T kept) the CUDA-core one
        if (e == cudaSuccess)
            e = a.bf16 ? kda::launch_chunk_intra_tc(a)
                       : (a.tmat ? kda::launch_chunk_intra(a) : kda::launch_chunk_intra_f32_tc(a));
        if (e == cudaSuccess) e = mark_stage(2, a.stream);
        if (e == cudaSuccess)
            e = a.bf16 ? kda::launch_chunk_inter_tc(a)
                       : (a.tmat ? kda::launch_chunk_inter(a) : kda::launch_chunk_inter_f32_tc(a));
    }
    if (e == cudaSuccess) e = mark_stage(3, a.stream);
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "kda_chunk_fwd launch failed: %s", cudaGetErrorString(e));
    return ok();
}

static kda_status recurrent_step_impl(const void* q, const void* k, const void* v, const float* log_alpha,
                                      const float* beta, float* state_inout, int B, int H, int dk, int dv,
                                      kda_dtype dtype, kda_gate gate, void* o, void* stream) {
    if (dtype != KDA_F32 && dtype != KDA_BF16) return fail(KDA_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (gate != KDA_GATE_CHANNEL && gate != KDA_GATE_HEAD && gate != KDA_GATE_NONE)
        return fail(KDA_ERR_INVALID_ARG, "unknown gate kind %d", (int)gate);
    if (B < 0 || H <= 0 || dk <= 0 || dv <= 0)
        return fail(KDA_ERR_INVALID_ARG, "bad sizes B=%d H=%d dk=%d dv=%d", B, H, dk, dv);
    if (!supported_dim(dk) || !supported_dim(dv))
        return fail(KDA_ERR_UNSUPPORTED, "head sizes dk=%d dv=%d not in {64, 128}", dk, dv);
    if ((size_t)B * H * dk * dv >= (size_t)1 << 40)
        return fail(KDA_ERR_UNSUPPORTED, "state too large");
    if (B > 0) {
        if (!q || !k || !v || !beta || !state_inout || !o || (gate != KDA_GATE_NONE && !log_alpha))
            return fail(KDA_ERR_INVALID_ARG, "null pointer");
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state_inout) || !aligned16(o) ||
            (gate == KDA_GATE_CHANNEL && !aligned16(log_alpha)))
            return fail(KDA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
        const char* s0 = (const char*)state_inout;
        const char* o0 = (const char*)o;
        const size_t sb = (size_t)B * H * dk * dv * sizeof(float);
        const size_t ob = (size_t)B * H * dv * (dtype == KDA_BF16 ? 2 : 4);
        if (o0 < s0 + sb && s0 < o0 + ob) return fail(KDA_ERR_INVALID_ARG, "o aliases state_inout");
    }
    kda::DecodeArgs a{};
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.state = state_inout; a.o = o;
    a.B = B; a.H = H; a.dk = dk; a.dv = dv;
    a.gate = (int)gate;
    a.bf16 = dtype == KDA_BF16;
    a.scale = 1.0f / sqrtf((float)dk);
    a.stream = static_cast<cudaStream_t>(stream);
    const cudaError_t e = kda::launch_decode(a);
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "kda_recurrent_step launch failed: %s", cudaGetErrorString(e));
    return ok();
}

kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const float* log_alpha,
                         const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                         int B, int T, int H, int dk, int dv, int num_seqs, kda_dtype dtype,
                         void* o, float* final_state, void* workspace, size_t workspace_bytes,
                         void* stream) {
    return chunk_fwd_impl(q, k, v, log_alpha, beta, initial_state, cu_seqlens, B, T, H, dk, dv, num_seqs,
                          dtype, KDA_GATE_CHANNEL, o, final_state, workspace, workspace_bytes, stream);
}

kda_status kda_chunk_fwd_gated(const void* q, const void* k, const void* v, const float* log_alpha,
                               const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                               int B, int T, int H, int dk, int dv, int num_seqs, kda_dtype dtype,
                               kda_gate gate, void* o, float* final_state, void* workspace,
                               size_t workspace_bytes, void* stream) {
    return chunk_fwd_impl(q, k, v, log_alpha, beta, initial_state, cu_seqlens, B, T, H, dk, dv, num_seqs,
                          dtype, gate, o, final_state, workspace, workspace_bytes, stream);
}

kda_status kda_recurrent_step(const void* q, const void* k, const void* v, const float* log_alpha,
                              const float* beta, float* state_inout, int B, int H, int dk, int dv,
                              kda_dtype dtype, void* o, void* stream) {
    return recurrent_step_impl(q, k, v, log_alpha, beta, state_inout, B, H, dk, dv, dtype, KDA_GATE_CHANNEL,
                               o, stream);
}

kda_status kda_recurrent_step_gated(const void* q, const void* k, const void* v, const float* log_alpha,
                                    const float* beta, float* state_inout, int B, int H, int dk, int dv,
                                    kda_dtype dtype, kda_gate gate, void* o, void* stream) {
    return recurrent_step_impl(q, k, v, log_alpha, beta, state_inout, B, H, dk, dv, dtype, gate, o, stream);
}

size_t kda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs, int varlen,
                                    kda_dtype dtype) {
    BwdLayout L;
    if (!bwd_layout(B, T, H, dk, dv, num_seqs, varlen != 0, dtype, L)) return 0;
    return L.total;
}

static kda_status chunk_bwd_impl(const void* q, const void* k, const void* v, const float* log_alpha,
                                 const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                                 const void* d_o, const float* d_final_state, int B, int T, int H, int dk,
                                 int dv, int num_seqs, kda_dtype dtype, kda_gate gate, void* dq, void* dk_out,
                                 void* dv_out, float* dlog_alpha, float* dbeta, float* d_initial_state,
                                 void* workspace, size_t workspace_bytes, void* stream, bool saved = false) {
    if (dtype != KDA_F32 && dtype != KDA_BF16) return fail(KDA_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (gate != KDA_GATE_CHANNEL && gate != KDA_GATE_HEAD && gate != KDA_GATE_NONE)
        return fail(KDA_ERR_INVALID_ARG, "unknown gate kind %d", (int)gate);
    if (B < 0 || T < 0 || H <= 0) return fail(KDA_ERR_INVALID_ARG, "bad sizes B=%d T=%d H=%d", B, T, H);
    if (dk <= 0 || dv <= 0) return fail(KDA_ERR_INVALID_ARG, "bad head sizes dk=%d dv=%d", dk, dv);
    if (!supported_dim(dk) || !supported_dim(dv))
        return fail(KDA_ERR_UNSUPPORTED, "head sizes dk=%d dv=%d not in {64, 128}", dk, dv);
    const bool varlen = cu_seqlens != nullptr;
    if (varlen && B != 1) return fail(KDA_ERR_INVALID_ARG, "cu_seqlens requires B == 1 (got B=%d)", B);
    if (varlen && num_seqs < 0) return fail(KDA_ERR_INVALID_ARG, "num_seqs=%d < 0", num_seqs);
    const int N = varlen ? num_seqs : B;
    const size_t tokens = varlen ? (size_t)T : (size_t)B * T;
    if (tokens * (size_t)H * (size_t)(dk > dv ? dk : dv) >= (size_t)1 << 31)
        return fail(KDA_ERR_UNSUPPORTED, "B*T*H*d = %zu elements exceeds 2^31", tokens * H * (dk > dv ? dk : dv));
    if (tokens > 0) {
        if (!q || !k || !v || !beta || !d_o || !dq || !dk_out || !dv_out || !dbeta ||
            (gate != KDA_GATE_NONE && (!log_alpha || !dlog_alpha)))
            return fail(KDA_ERR_INVALID_ARG, "null input/output pointer");
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(d_o) ||
            (gate == KDA_GATE_CHANNEL && !aligned16(log_alpha)))
            return fail(KDA_ERR_INVALID_ARG, "q/k/v/log_alpha/d_o must be 16-byte aligned");
    }
    BwdLayout L;
    if (!bwd_layout(B, T, H, dk, dv, num_seqs, varlen, dtype, L))
        return fail(KDA_ERR_INVALID_ARG, "invalid sizes for the workspace layout");
    if (!workspace) return fail(KDA_ERR_WORKSPACE, "workspace is null (need %zu bytes)", L.total);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(KDA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    if (workspace_bytes < L.total)
        return fail(KDA_ERR_WORKSPACE, "workspace has %zu bytes, need %zu", workspace_bytes, L.total);

    char* ws = static_cast<char*>(workspace);
    kda::ChunkArgs a{};
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.initial_state = initial_state; a.cu_seqlens = cu_seqlens;
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv; a.num_seqs = N;
    a.gate = (int)gate;
    a.bf16 = dtype == KDA_BF16;
    a.scale = 1.0f / sqrtf((float)dk);
    a.ws_header = workspace;
    a.chunk_offsets = reinterpret_cast<int32_t*>(ws + L.base.offsets_off);
    a.records = ws + L.base.records_off;
    a.max_chunks = L.base.max_chunks;
    a.fixed_chunks_per_seq = L.base.chunks_per_seq;
    a.stream = static_cast<cudaStream_t>(stream);
    a.tmat = a.bf16 ? nullptr : reinterpret_cast<float*>(ws + L.tmat_off);
    a.bwd_tiles = a.bf16 ? static_cast<void*>(ws + L.tiles_off) : nullptr;
    a.bwd_flags = a.bf16 ? reinterpret_cast<int*>(ws + L.flags_off) : nullptr;
    a.states = reinterpret_cast<float*>(ws + L.states_off);
    a.d_o = d_o; a.d_final_state = d_final_state;
    a.dq = dq; a.dk_out = dk_out; a.dv_out = dv_out;
    a.dlog_alpha = dlog_alpha; a.dbeta = dbeta; a.d_initial_state = d_initial_state;
    a.dS_end = reinterpret_cast<float*>(ws + L.dS_off);
    a.dU = reinterpret_cast<float*>(ws + L.dU_off);
    a.scratch = reinterpret_cast<float*>(ws + L.scratch_off);
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "device query failed: %s", cudaGetErrorString(e));
    a.bwd_ctas = L.ctas < 2 * sms ? L.ctas : 2 * sms;   // two resident per SM

    // forward recomputation (the records, T and the chunk-start states: fp16
    // records on the tensor cores for bf16 inputs, fp32 ones on CUDA cores for
    // fp32 inputs) unless kda_chunk_fwd_save left them in this workspace, then
    // the reversed pass over chunks, then the per-chunk gradients
    const bool marks = g_stage_event_count >= 7;   // the backward records all seven or none
    auto mark = [&](int i) { return marks ? mark_stage(i, a.stream) : cudaSuccess; };
    e = mark(0);
    if (e == cudaSuccess && !saved) e = kda::launch_chunk_prep(a);
    if (e == cudaSuccess) e = mark(1);
    if (e == cudaSuccess && !saved) e = a.bf16 ? kda::launch_chunk_intra_tc(a) : kda::launch_chunk_intra(a);
    if (e == cudaSuccess) e = mark(2);
    if (e == cudaSuccess && !saved) e = a.bf16 ? kda::launch_chunk_inter_tc(a) : kda::launch_chunk_inter(a);
    if (e == cudaSuccess) e = mark(3);
    // the reversed chain reads the fp16 tensor-core records (bf16) or the fp32
    // ones; for bf16 the products over the value dimension are formed on the
    // tensor cores too, and the per-chunk gradient kernel reads no record
    if (e == cudaSuccess) e = a.bf16 ? kda::launch_chunk_bwd_inter_tc(a) : kda::launch_chunk_bwd_inter(a);
    if (e == cudaSuccess) e = mark(4);
    if (a.bf16) {
        a.vside = reinterpret_cast<float*>(ws + L.vside_off);
        if (e == cudaSuccess) e = kda::launch_chunk_bwd_vside_tc(a);
        if (e == cudaSuccess) e = kda::launch_chunk_bwd_tchain_tc(a);
        if (e == cudaSuccess) e = kda::launch_chunk_bwd_split_tc(a);
    }
    if (e == cudaSuccess) e = mark(5);
    if (e == cudaSuccess) e = kda::launch_chunk_bwd_intra(a);
    if (e == cudaSuccess) e = mark(6);
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "kda_chunk_bwd launch failed: %s", cudaGetErrorString(e));
    return ok();
}

kda_status kda_chunk_bwd(const void* q, const void* k, const void* v, const float* log_alpha,
                         const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                         const void* d_o, const float* d_final_state, int B, int T, int H, int dk, int dv,
                         int num_seqs, kda_dtype dtype, void* dq, void* dk_out, void* dv_out,
                         float* dlog_alpha, float* dbeta, float* d_initial_state, void* workspace,
                         size_t workspace_bytes, void* stream) {
    return chunk_bwd_impl(q, k, v, log_alpha, beta, initial_state, cu_seqlens, d_o, d_final_state, B, T, H, dk,
                          dv, num_seqs, dtype, KDA_GATE_CHANNEL, dq, dk_out, dv_out, dlog_alpha, dbeta,
                          d_initial_state, workspace, workspace_bytes, stream);
}

kda_status kda_chunk_bwd_gated(const void* q, const void* k, const void* v, const float* log_alpha,
                               const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                               const void* d_o, const float* d_final_state, int B, int T, int H, int dk,
                               int dv, int num_seqs, kda_dtype dtype, kda_gate gate, void* dq, void* dk_out,
                               void* dv_out, float* dlog_alpha, float* dbeta, float* d_initial_state,
                               void* workspace, size_t workspace_bytes, void* stream) {
    return chunk_bwd_impl(q, k, v, log_alpha, beta, initial_state, cu_seqlens, d_o, d_final_state, B, T, H, dk,
                          dv, num_seqs, dtype, gate, dq, dk_out, dv_out, dlog_alpha, dbeta, d_initial_state,
                          workspace, workspace_bytes, stream);
}

int kda_chunk_fwd_plan(int B, int T, int H, int dk, int dv, int num_seqs, int varlen, kda_dtype dtype,
                       size_t workspace_bytes) {
    WsLayout L;
    if (!ws_layout(B, T, H, dk, dv, num_seqs, varlen != 0, dtype, L)) return -1;
    const int N = varlen ? num_seqs : B;
    const int fused = chunk_fwd_fused(N, varlen != 0, dtype, L, workspace_bytes);
    if (workspace_bytes < L.total && !fused) return -1;
    return fused;
}

size_t kda_chunk_fwd_fused_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs, int varlen,
                                          kda_dtype dtype) {
    WsLayout L;
    if (dtype != KDA_BF16 || !ws_layout(B, T, H, dk, dv, num_seqs, varlen != 0, dtype, L)) return 0;
    return fused_ws_bytes(varlen ? num_seqs : B, varlen != 0, L);
}

kda_status kda_chunk_fwd_save(const void* q, const void* k, const void* v, const float* log_alpha,
                              const float* beta, const float* initial_state, const int32_t* cu_seqlens, int B,
                              int T, int H, int dk, int dv, int num_seqs, kda_dtype dtype, kda_gate gate,
                              void* o, float* final_state, void* workspace, size_t workspace_bytes,
                              void* stream) {
    return chunk_fwd_impl(q, k, v, log_alpha, beta, initial_state, cu_seqlens, B, T, H, dk, dv, num_seqs,
                          dtype, gate, o, final_state, workspace, workspace_bytes, stream, /*save=*/true);
}

kda_status kda_chunk_bwd_saved(const void* q, const void* k, const void* v, const float* log_alpha,
                               const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                               const void* d_o, const float* d_final_state, int B, int T, int H, int dk,
                               int dv, int num_seqs, kda_dtype dtype, kda_gate gate, void* dq, void* dk_out,
                               void* dv_out, float* dlog_alpha, float* dbeta, float* d_initial_state,
                               void* workspace, size_t workspace_bytes, void* stream) {
    return chunk_bwd_impl(q, k, v, log_alpha, beta, initial_state, cu_seqlens, d_o, d_final_state, B, T, H, dk,
                          dv, num_seqs, dtype, gate, dq, dk_out, dv_out, dlog_alpha, dbeta, d_initial_state,
                          workspace, workspace_bytes, stream, /*saved=*/true);
}

kda_status kda_workspace_status(const void* workspace, size_t workspace_bytes, void* stream) {
    if (!workspace || workspace_bytes < (size_t)kda::kHeaderBytes)
        return fail(KDA_ERR_WORKSPACE, "workspace missing or smaller than its header");
    int words[3] = {0, 0, 0};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(words, workspace, sizeof(words), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "reading workspace status: %s", cudaGetErrorString(e));
    const int st = words[0] != 0 ? words[0] : words[2];
    if (st == kda::kStatusOk) return ok();
    if (st == kda::kStatusBadSeqlens) return fail(KDA_ERR_BAD_SEQLENS, "cu_seqlens rejected on the device");
    if (st == kda::kStatusTimeout) return fail(KDA_ERR_TIMEOUT, "a bounded wait inside a kernel gave up");
    if (st == kda::kStatusInternal) return fail(KDA_ERR_CUDA, "a kernel found its shared memory misaligned");
    if (st == kda::kStatusRange)
        return fail(KDA_ERR_RANGE, "an intermediate exceeded the fp16 range of the bf16 path (use fp32 inputs)");
    return fail(KDA_ERR_CUDA, "unknown device status %d", st);
}

kda_status kda_set_stage_events(void* const* events, int count) {
    if (!events) {
        g_stage_event_count = 0;
        return ok();
    }
    if (count < 4) return fail(KDA_ERR_INVALID_ARG, "need at least 4 events, got %d", count);
    const int n = count < kMaxStageEvents ? count : kMaxStageEvents;
    for (int i = 0; i < n; ++i)
        if (!events[i]) return fail(KDA_ERR_INVALID_ARG, "event %d is null", i);
    for (int i = 0; i < n; ++i) g_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
    g_stage_event_count = n;
    return ok();
}

kda_status kda_debug_drop_copy(long long wait_cycles) {
    if (wait_cycles < 0) return fail(KDA_ERR_INVALID_ARG, "wait_cycles=%lld < 0", wait_cycles);
    g_debug_drop_cap = wait_cycles;
    return ok();
}

const char* kda_last_error(void) { return g_last_error.c_str(); }

const char* kda_version(void) { return "kda-b200 0.1.0 sm_100a"; }

}  // extern "C"
