// specdec_api.cu — the C-ABI (include/specdec.h): argument checks, workspace
// layout, grid sizing and kernel launches.
//
// Workspace layout (byte offsets).  The words that must be zero when a call
// starts sit at a fixed place, so a workspace initialised once serves calls
// of any shape; each call returns those words to zero before it ends.
//   [0, 256 KiB)            top-8 thresholds, one word per row (first 65536 rows)
//   then                    streaming-pass partials, one slot per chunk
//   then (rejection only)   per-request RejState, per-chunk and per-unit masses
//                           of row h
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>

#include "../../include/specdec.h"
#include "verify_pass1.cuh"
#include "verify_resample.cuh"
#include "verify_stats.cuh"
#include "verify_ngram.cuh"

namespace specdec {
namespace {

constexpr size_t kThetaBase = 0;
constexpr size_t kPartialBase = kThetaBase + static_cast<size_t>(kThetaRows) * sizeof(unsigned);

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Layout {
    int64_t nv = 0, nv_full = 0, cpr = 0, NC = 0, cpr2 = 0;
    size_t partials1 = 0, state = 0, masses = 0, units = 0, row_stat = 0, chunk_stats = 0, total = 0;
};

// Layout of one call.  `vec` = elements per vector (1 on the scalar path),
// `slot1` = bytes of pass-1 partials per chunk.
Layout make_layout(int64_t rows, int rows_per_req, int B, int V, int vec, size_t slot1, bool rejection,
                   int u = kU) {
    Layout L;
    L.total = kPartialBase;
    if (rows <= 0 || V <= 0) return L;  // nothing streamed: only the fixed area
    L.nv = (V + vec - 1) / vec;
    L.nv_full = V / vec;
    L.cpr = chunks_per_row(L.nv_full, vec, u);
    L.NC = rows * L.cpr;
    L.partials1 = kPartialBase;
    size_t end = L.partials1 + static_cast<size_t>(L.NC) * slot1;
    if (rejection) {
        L.state = align_up(end, 256);
        end = L.state + static_cast<size_t>(B) * sizeof(RejState);
        L.cpr2 = chunks_per_row(L.nv_full, vec, kU2);
        L.masses = align_up(end, 256);
        end = L.masses + static_cast<size_t>(B) * static_cast<size_t>(L.cpr2) * sizeof(double2);
        L.units = align_up(end, 256);
        end = L.units + static_cast<size_t>(B) * static_cast<size_t>(L.cpr2) *
                            static_cast<size_t>(units_per_chunk(vec)) * sizeof(double2);
        // draft statistics (fixed layout: rows - B = B k draft rows)
        L.row_stat = align_up(end, 256);
        end = L.row_stat + static_cast<size_t>(rows) * sizeof(RowStat);
        L.chunk_stats = align_up(end, 256);
        end = L.chunk_stats + static_cast<size_t>(rows - B) * static_cast<size_t>(L.cpr2) * sizeof(double2);
    }
    (void)rows_per_req;
    L.total = align_up(end, 256);
    return L;
}

int elem_size(specdec_dtype dt) { return dt == SPECDEC_BF16 ? 2 : 4; }
int vec_elems(specdec_dtype dt) { return dt == SPECDEC_BF16 ? 8 : 4; }

constexpr int kMaxDevices = 64;

// specdec_set_prefetch_inputs: whether the argmax streaming pass may read its
// rows before the previous kernel of the stream has finished.
std::atomic<int> g_prefetch_inputs{0};

bool vector_path_ok(const void* p, int64_t stride, int esize) {
    return (reinterpret_cast<uintptr_t>(p) % 16 == 0) && ((stride * esize) % 16 == 0);
}

bool rows_fit(int64_t rows, int64_t row_stride, int V) {
    // Every element offset must fit comfortably in 63 bits.
    return row_stride >= V && row_stride <= (int64_t(1) << 40) && rows * row_stride < (int64_t(1) << 52);
}

// Launch with programmatic stream serialisation: the kernel may be scheduled
// while the previous kernel of the stream drains; it waits (griddepcontrol)
// before touching global memory, so stream order is kept.
template <class Kernel, class Params>
cudaError_t launch_pdl(Kernel fn, dim3 grid, int dyn, cudaStream_t stream, const Params& P, int block = NT) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(static_cast<unsigned>(block));
    cfg.dynamicSmemBytes = static_cast<size_t>(dyn);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fn, P);
}

// The streaming pass (one CTA per chunk; trees stream like greedy argmax),
// then the request epilogues (one CTA per request).
template <class Tag, int VEC, int MODE>
specdec_status launch_pass1(Pass1Params P, cudaStream_t stream) {
    constexpr int STREAM_MODE = MODE == MODE_TREE ? MODE_ARGMAX : MODE;
    if (P.R > 0x7fffffff || P.cpr > 65535) return SPECDEC_ERR_UNSUPPORTED;  // grid limits
    const dim3 grid(static_cast<unsigned>(P.R), static_cast<unsigned>(P.cpr));
    if (launch_pdl(verify_pass1_kernel<Tag, VEC, STREAM_MODE>, grid, 0, stream, P) != cudaSuccess)
        return SPECDEC_ERR_CUDA;
    if constexpr (MODE == MODE_TOP8) {
        const int rows = P.k + 1 < kTop8EpiWarps ? P.k + 1 : kTop8EpiWarps;  // a warp per row
        if (launch_pdl(verify_top8_epilogue_kernel<Tag>, dim3(static_cast<unsigned>(P.B)), 0, stream, P, 32 * rows) !=
            cudaSuccess)
            return SPECDEC_ERR_CUDA;
    } else {
        if (launch_pdl(verify_epilogue_kernel<Tag, MODE>, dim3(static_cast<unsigned>(P.B)), 0, stream, P) !=
            cudaSuccess)
            return SPECDEC_ERR_CUDA;
    }
    return cudaGetLastError() == cudaSuccess ? SPECDEC_OK : SPECDEC_ERR_CUDA;
}

// The chunk masses of row h (one CTA per chunk), then the token search (one
// CTA per request).
template <class Tag, int VEC>
specdec_status launch_pass2(Pass2Params P, cudaStream_t stream) {
    if (P.cpr > 65535) return SPECDEC_ERR_UNSUPPORTED;  // grid limit
    const dim3 grid(static_cast<unsigned>(P.B), static_cast<unsigned>(P.cpr));
    if (launch_pdl(verify_resample_kernel<Tag, VEC>, grid, 0, stream, P) != cudaSuccess) return SPECDEC_ERR_CUDA;
    const unsigned search_ctas = static_cast<unsigned>((P.B + NWARPS - 1) / NWARPS);  // a warp per request
    if (launch_pdl(verify_resample_epilogue_kernel<Tag, VEC>, dim3(search_ctas), 0, stream, P) != cudaSuccess)
        return SPECDEC_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? SPECDEC_OK : SPECDEC_ERR_CUDA;
}

template <int MODE>
specdec_status dispatch_pass1(specdec_dtype dt, bool vec, Pass1Params P, cudaStream_t s) {
    if (dt == SPECDEC_BF16)
        return vec ? launch_pass1<BF16Tag, 8, MODE>(P, s) : launch_pass1<BF16Tag, 1, MODE>(P, s);
    return vec ? launch_pass1<F32Tag, 4, MODE>(P, s) : launch_pass1<F32Tag, 1, MODE>(P, s);
}

specdec_status dispatch_pass2(specdec_dtype dt, bool vec, Pass2Params P, cudaStream_t s) {
    if (dt == SPECDEC_BF16) return vec ? launch_pass2<BF16Tag, 8>(P, s) : launch_pass2<BF16Tag, 1>(P, s);
    return vec ? launch_pass2<F32Tag, 4>(P, s) : launch_pass2<F32Tag, 1>(P, s);
}

// AdaSD statistics: the chunk sums of every draft row, then a warp per
// (request, position).
template <class Tag, int VEC>
specdec_status launch_stats(StatsParams S, cudaStream_t stream) {
    const int64_t rows = static_cast<int64_t>(S.B) * S.k;
    if (S.cpr > 65535 || rows > 0x7fffffff) return SPECDEC_ERR_UNSUPPORTED;
    const dim3 grid(static_cast<unsigned>(rows), static_cast<unsigned>(S.cpr));
    if (launch_pdl(verify_stats_kernel<Tag, VEC>, grid, 0, stream, S) != cudaSuccess) return SPECDEC_ERR_CUDA;
    if (launch_pdl(verify_stats_epilogue_kernel, dim3(static_cast<unsigned>((rows + NWARPS - 1) / NWARPS)), 0,
                   stream, S) != cudaSuccess)
        return SPECDEC_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? SPECDEC_OK : SPECDEC_ERR_CUDA;
}

specdec_status dispatch_stats(specdec_dtype dt, bool vec, StatsParams S, cudaStream_t s) {
    if (dt == SPECDEC_BF16) return vec ? launch_stats<BF16Tag, 8>(S, s) : launch_stats<BF16Tag, 1>(S, s);
    return vec ? launch_stats<F32Tag, 4>(S, s) : launch_stats<F32Tag, 1>(S, s);
}

bool dtype_ok(specdec_dtype dt) { return dt == SPECDEC_F32 || dt == SPECDEC_BF16; }

// Pass-1 partial bytes per chunk: one argmax key per warp, 8 keys per warp
// (top-8), or one (max, sum) pair per warp (softmax).
constexpr size_t kArgmaxChunkBytes = NWARPS * sizeof(uint64_t);
constexpr size_t kTop8ChunkBytes = NWARPS * 8 * sizeof(uint64_t);
constexpr size_t kSoftmaxChunkBytes = NWARPS * sizeof(SoftmaxPartial);
size_t slot_bytes(specdec_mode mode) {
    if (mode == SPECDEC_MODE_GREEDY) return kArgmaxChunkBytes > kTop8ChunkBytes ? kArgmaxChunkBytes : kTop8ChunkBytes;
    if (mode == SPECDEC_MODE_REJECTION) return kSoftmaxChunkBytes;
    return kArgmaxChunkBytes;
}

specdec_status check_ws(void* ws, size_t ws_bytes, size_t need) {
    if (ws == nullptr || reinterpret_cast<uintptr_t>(ws) % 16 != 0) return SPECDEC_ERR_WORKSPACE;
    if (ws_bytes < need) return SPECDEC_ERR_WORKSPACE;
    return SPECDEC_OK;
}

void fill_common(Pass1Params& P, const void* logits, int64_t row_stride, int V, const Layout& L, int64_t rows,
                 int rows_per_req, int B, void* ws) {
    memset(&P, 0, sizeof(P));
    P.prefetch_inputs = g_prefetch_inputs.load(std::memory_order_relaxed);
    char* base = static_cast<char*>(ws);
    P.logits = logits;
    P.row_stride = row_stride;
    P.V = V;
    P.nv_full = static_cast<int>(L.nv_full);
    P.R = rows;
    P.cpr = static_cast<int>(L.cpr);
    P.NC = static_cast<uint64_t>(L.NC);
    P.rows_per_req = rows_per_req;
    P.B = B;
    P.theta_row = reinterpret_cast<unsigned*>(base + kThetaBase);
    P.partials = base + L.partials1;
}

}  // namespace
}  // namespace specdec

namespace specdec {
namespace {

// Every check specdec_verify_greedy makes before it launches anything, the
// workspace's aside (B == 0 passes: such a call does nothing).
specdec_status greedy_args_status(const void* logits, specdec_dtype dtype, int64_t row_stride,
                                  const int32_t* draft_tokens, int B, int k, int V, const int32_t* accept_len,
                                  const int32_t* out_tokens, int topk, const int32_t* topk_ids,
                                  const float* topk_vals) {
    if (!dtype_ok(dtype)) return SPECDEC_ERR_UNSUPPORTED;
    if (B < 0 || B > SPECDEC_MAX_B || k < 0 || k > SPECDEC_MAX_K || V < 1 || V > SPECDEC_MAX_V)
        return SPECDEC_ERR_INVALID_ARG;
    if (topk < 0 || topk > SPECDEC_MAX_TOPK) return SPECDEC_ERR_INVALID_ARG;
    if (B == 0) return SPECDEC_OK;
    if (!rows_fit(static_cast<int64_t>(B) * (k + 1), row_stride, V)) return SPECDEC_ERR_INVALID_ARG;
    if (logits == nullptr || accept_len == nullptr || out_tokens == nullptr) return SPECDEC_ERR_INVALID_ARG;
    if (k > 0 && draft_tokens == nullptr) return SPECDEC_ERR_INVALID_ARG;
    if (topk > 0 && (topk_ids == nullptr || topk_vals == nullptr)) return SPECDEC_ERR_INVALID_ARG;
    return SPECDEC_OK;
}

// Greedy verification over `rows` logit rows: the fixed layout (offsets null,
// k drafts per request, rows = B (k + 1)) or the packed one (offsets [B+1],
// k = the bound on every request's count, rows = B + total drafts).
specdec_status greedy_impl(const void* logits, specdec_dtype dtype, int64_t row_stride, const int32_t* draft_tokens,
                           const int32_t* offsets, int64_t total, int B, int k, int V, int32_t* accept_len,
                           int32_t* out_tokens, int topk, int32_t* topk_ids, float* topk_vals, int64_t* counters,
                           void* ws, size_t ws_bytes, cudaStream_t s) {
    const int64_t rows = offsets ? B + total : static_cast<int64_t>(B) * (k + 1);
    if (!rows_fit(rows, row_stride, V)) return SPECDEC_ERR_INVALID_ARG;
    if (logits == nullptr || accept_len == nullptr || out_tokens == nullptr) return SPECDEC_ERR_INVALID_ARG;
    if (total > 0 && draft_tokens == nullptr) return SPECDEC_ERR_INVALID_ARG;
    if (topk > 0 && (topk_ids == nullptr || topk_vals == nullptr)) return SPECDEC_ERR_INVALID_ARG;
    const bool vec = vector_path_ok(logits, row_stride, elem_size(dtype));
    const int ve = vec ? vec_elems(dtype) : 1;
    const Layout L = make_layout(rows, k + 1, B, V, ve, topk > 0 ? kTop8ChunkBytes : kArgmaxChunkBytes, false,
                                 mode_u(topk > 0 ? MODE_TOP8 : MODE_ARGMAX));
    specdec_status st = check_ws(ws, ws_bytes, L.total);
    if (st != SPECDEC_OK) return st;
    Pass1Params P;
    fill_common(P, logits, row_stride, V, L, rows, k + 1, B, ws);
    P.drafts = draft_tokens;
    P.k = k;
    P.draft_offsets = offsets;
    P.total_drafts = total;
    P.counters = counters;
    P.accept_len = accept_len;
    P.out_tokens = out_tokens;
    P.topk = topk;
    P.topk_ids = topk_ids;
    P.topk_vals = topk_vals;
    if (topk > 0) return dispatch_pass1<MODE_TOP8>(dtype, vec, P, s);
    if (static_cast<int64_t>(k + 1) * V * elem_size(dtype) <= kSmallRequestBytes) {
        // small requests: the whole verification in one launch, a CTA per request
        cudaError_t e;
        if (dtype == SPECDEC_BF16)
            e = vec ? launch_pdl(verify_small_greedy_kernel<BF16Tag, 8>, dim3(static_cast<unsigned>(B)), 0, s, P)
                    : launch_pdl(verify_small_greedy_kernel<BF16Tag, 1>, dim3(static_cast<unsigned>(B)), 0, s, P);
        else
            e = vec ? launch_pdl(verify_small_greedy_kernel<F32Tag, 4>, dim3(static_cast<unsigned>(B)), 0, s, P)
                    : launch_pdl(verify_small_greedy_kernel<F32Tag, 1>, dim3(static_cast<unsigned>(B)), 0, s, P);
        if (e != cudaSuccess) return SPECDEC_ERR_CUDA;
        return cudaGetLastError() == cudaSuccess ? SPECDEC_OK : SPECDEC_ERR_CUDA;
    }
    return dispatch_pass1<MODE_ARGMAX>(dtype, vec, P, s);
}

// Rejection-sampling verification, fixed or packed layout as greedy_impl.
specdec_status rejection_impl(const void* target_logits, specdec_dtype dtype, int64_t row_stride,
                              const float* draft_probs, int64_t q_row_stride, const int32_t* draft_tokens,
                              const int32_t* offsets, int64_t total, int B, int k, int V, float temperature,
                              uint64_t seed, uint64_t offset, int32_t* accept_len, int32_t* out_tokens,
                              float* p_draft_out, int64_t* counters, double* entropy, double* js, void* ws,
                              size_t ws_bytes, cudaStream_t s, uint32_t req_base = 0) {
    if (!(isnormal(temperature) && temperature > 0.0f)) return SPECDEC_ERR_INVALID_ARG;
    const int64_t rows = offsets ? B + total : static_cast<int64_t>(B) * (k + 1);
    if (!rows_fit(rows, row_stride, V)) return SPECDEC_ERR_INVALID_ARG;
    if (target_logits == nullptr || accept_len == nullptr || out_tokens == nullptr) return SPECDEC_ERR_INVALID_ARG;
    if (total > 0 && (draft_tokens == nullptr || draft_probs == nullptr)) return SPECDEC_ERR_INVALID_ARG;
    if (total > 0 && !rows_fit(total, q_row_stride, V)) return SPECDEC_ERR_INVALID_ARG;
    const bool vec = vector_path_ok(target_logits, row_stride, elem_size(dtype)) &&
                     (total == 0 || vector_path_ok(draft_probs, q_row_stride, 4));
    const int ve = vec ? vec_elems(dtype) : 1;
    const Layout L = make_layout(rows, k + 1, B, V, ve, kSoftmaxChunkBytes, true);
    specdec_status st = check_ws(ws, ws_bytes, L.total);
    if (st != SPECDEC_OK) return st;
    const double invT_d = 1.0 / static_cast<double>(temperature);
    RejState* state = reinterpret_cast<RejState*>(static_cast<char*>(ws) + L.state);
    Pass1Params P;
    fill_common(P, target_logits, row_stride, V, L, rows, k + 1, B, ws);
    P.drafts = draft_tokens;
    P.k = k;
    P.draft_offsets = offsets;
    P.total_drafts = total;
    P.counters = counters;
    P.accept_len = accept_len;
    P.out_tokens = out_tokens;
    P.q = draft_probs;
    P.q_stride = q_row_stride;
    P.invT = static_cast<float>(invT_d);
    P.log2e_invT = static_cast<float>(invT_d * 1.4426950408889634);  // log2(e) / T, rounded once
    P.invT_d = invT_d;
    P.seed = seed;
    P.offset = offset;
    P.p_draft_out = p_draft_out;
    P.state = state;
    P.req_base = req_base;
    const bool stats = entropy != nullptr && offsets == nullptr && k > 0;
    P.row_stat = stats ? reinterpret_cast<RowStat*>(static_cast<char*>(ws) + L.row_stat) : nullptr;
    st = dispatch_pass1<MODE_SOFTMAX>(dtype, vec, P, s);
    if (st != SPECDEC_OK) return st;
    Pass2Params Q;
    memset(&Q, 0, sizeof(Q));
    Q.logits = target_logits;
    Q.row_stride = row_stride;
    Q.q = draft_probs;
    Q.q_stride = q_row_stride;
    Q.V = V;
    Q.nv_full = static_cast<int>(L.nv_full);
    Q.cpr = static_cast<int>(L.cpr2);
    Q.B = B;
    Q.k = k;
    Q.invT = static_cast<float>(invT_d);
    Q.log2e_invT = P.log2e_invT;
    Q.seed = seed;
    Q.offset = offset;
    Q.req_base = req_base;
    Q.state = state;
    Q.chunk_mass = reinterpret_cast<double2*>(static_cast<char*>(ws) + L.masses);
    Q.unit_mass = reinterpret_cast<double2*>(static_cast<char*>(ws) + L.units);
    Q.out_tokens = out_tokens;
    st = dispatch_pass2(dtype, vec, Q, s);
    if (st != SPECDEC_OK || !stats) return st;
    StatsParams S;
    memset(&S, 0, sizeof(S));
    S.logits = target_logits;
    S.row_stride = row_stride;
    S.q = draft_probs;
    S.q_stride = q_row_stride;
    S.V = V;
    S.nv_full = static_cast<int>(L.nv_full);
    S.cpr = static_cast<int>(L.cpr2);
    S.B = B;
    S.k = k;
    S.log2e_invT = P.log2e_invT;
    S.state = state;
    S.row_stat = P.row_stat;
    S.chunk_stats = reinterpret_cast<double2*>(static_cast<char*>(ws) + L.chunk_stats);
    S.entropy = entropy;
    S.js = js;
    return dispatch_stats(dtype, vec, S, s);
}

// Vocabulary-sharded greedy: this shard's streaming pass, then its row keys.
template <class Tag, int VEC, int MODE>
specdec_status launch_shard_rows(Pass1Params P, cudaStream_t stream) {
    if (P.R > 0x7fffffff || P.cpr > 65535) return SPECDEC_ERR_UNSUPPORTED;
    const dim3 grid(static_cast<unsigned>(P.R), static_cast<unsigned>(P.cpr));
    if (launch_pdl(verify_pass1_kernel<Tag, VEC, MODE>, grid, 0, stream, P) != cudaSuccess) return SPECDEC_ERR_CUDA;
    const int64_t per = MODE == MODE_TOP8 ? NWARPS : kShardRowsArgmax;
    const dim3 grid2(static_cast<unsigned>((P.R + per - 1) / per));
    if (launch_pdl(verify_shard_rows_kernel<Tag, MODE>, grid2, 0, stream, P) != cudaSuccess) return SPECDEC_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? SPECDEC_OK : SPECDEC_ERR_CUDA;
}

template <int MODE>
specdec_status dispatch_shard_rows(specdec_dtype dt, bool vec, Pass1Params P, cudaStream_t s) {
    if (dt == SPECDEC_BF16)
        return vec ? launch_shard_rows<BF16Tag, 8, MODE>(P, s) : launch_shard_rows<BF16Tag, 1, MODE>(P, s);
    return vec ? launch_shard_rows<F32Tag, 4, MODE>(P, s) : launch_shard_rows<F32Tag, 1, MODE>(P, s);
}

// Vocabulary-sharded rejection: the request state sits at a fixed place
// (every step finds it without the others' arguments), then the streaming
// partials, then the chunk and unit masses of this shard's part of row h.
Layout shard_rej_layout(int B, int k, int V_shard, int vec) {
    const int64_t rows = static_cast<int64_t>(B) * (k + 1);
    Layout L = make_layout(rows, k + 1, B, V_shard, vec, kSoftmaxChunkBytes, true);
    const size_t state = kPartialBase, state_end = align_up(state + static_cast<size_t>(B) * sizeof(RejState), 256);
    const size_t shift = state_end - L.partials1;  // move everything from the partials on past the state
    L.state = state;
    L.partials1 += shift;
    L.masses += shift;
    L.units += shift;
    L.row_stat += shift;
    L.chunk_stats += shift;
    L.total += shift;
    return L;
}

// Host checks of a packed-layout call.
bool ragged_args_ok(const int32_t* offsets, int B, int total, int max_k) {
    if (offsets == nullptr || total < 0 || max_k < 0 || max_k > SPECDEC_MAX_K) return false;
    return static_cast<int64_t>(total) <= static_cast<int64_t>(B) * max_k;
}

}  // namespace
}  // namespace specdec

using namespace specdec;

extern "C" {

int specdec_abi_version(void) { return SPECDEC_ABI_VERSION; }

const char* specdec_status_string(specdec_status s) {
    switch (s) {
        case SPECDEC_OK: return "ok";
        case SPECDEC_ERR_INVALID_ARG: return "invalid argument";
        case SPECDEC_ERR_UNSUPPORTED: return "unsupported dtype or mode";
        case SPECDEC_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case SPECDEC_ERR_CUDA: return "CUDA runtime error";
        case SPECDEC_ERR_TIMEOUT: return "timed out waiting on the device";
    }
    return "unknown status";
}

size_t specdec_workspace_size(specdec_mode mode, int B, int k_or_N, int V, specdec_dtype dtype) {
    if (!dtype_ok(dtype) || B < 0 || B > SPECDEC_MAX_B || V < 1 || V > SPECDEC_MAX_V) return 0;
    int rpr;
    if (mode == SPECDEC_MODE_TREE) {
        if (k_or_N < 0 || k_or_N + 1 > SPECDEC_MAX_TREE_NODES) return 0;
        rpr = k_or_N + 1;
    } else if (mode == SPECDEC_MODE_GREEDY || mode == SPECDEC_MODE_REJECTION) {
        if (k_or_N < 0 || k_or_N > SPECDEC_MAX_K) return 0;
        rpr = k_or_N + 1;
    } else {
        return 0;
    }
    const int64_t rows = static_cast<int64_t>(B) * rpr;
    const bool rej = mode == SPECDEC_MODE_REJECTION;
    // The larger of the vector and the scalar path's layouts.
    const Layout a = make_layout(rows, rpr, B, V, vec_elems(dtype), slot_bytes(mode), rej);
    const Layout b = make_layout(rows, rpr, B, V, 1, slot_bytes(mode), rej);
    return a.total > b.total ? a.total : b.total;
}

size_t specdec_workspace_size_shard(int rows, int V_shard, int topk, specdec_dtype dtype) {
    if (!dtype_ok(dtype) || rows < 0 || V_shard < 1 || V_shard > SPECDEC_MAX_V || topk < 0 || topk > SPECDEC_MAX_TOPK)
        return 0;
    const size_t slot = topk > 0 ? kTop8ChunkBytes : kArgmaxChunkBytes;
    const Layout a = make_layout(rows, 1, 1, V_shard, vec_elems(dtype), slot, false);
    const Layout b = make_layout(rows, 1, 1, V_shard, 1, slot, false);
    return a.total > b.total ? a.total : b.total;
}

specdec_status specdec_shard_greedy_rows(const void* logits, specdec_dtype dtype, int64_t row_stride, int rows,
                                         int V_shard, int vocab_offset, int topk, uint64_t* row_keys,
                                         float* row_vals, void* ws, size_t ws_bytes, struct CUstream_st* stream) {
    if (!dtype_ok(dtype)) return SPECDEC_ERR_UNSUPPORTED;
    if (rows < 0 || V_shard < 1 || V_shard > SPECDEC_MAX_V || topk < 0 || topk > SPECDEC_MAX_TOPK)
        return SPECDEC_ERR_INVALID_ARG;
    if (vocab_offset < 0 || static_cast<int64_t>(vocab_offset) + V_shard > SPECDEC_MAX_V) return SPECDEC_ERR_INVALID_ARG;
    if (rows == 0) return SPECDEC_OK;
    if (!rows_fit(rows, row_stride, V_shard)) return SPECDEC_ERR_INVALID_ARG;
    if (logits == nullptr || row_keys == nullptr || (topk > 0 && row_vals == nullptr)) return SPECDEC_ERR_INVALID_ARG;
    const bool vec = vector_path_ok(logits, row_stride, elem_size(dtype));
    const int ve = vec ? vec_elems(dtype) : 1;
    const Layout L = make_layout(rows, 1, 1, V_shard, ve, topk > 0 ? kTop8ChunkBytes : kArgmaxChunkBytes, false,
                                 mode_u(topk > 0 ? MODE_TOP8 : MODE_ARGMAX));
    specdec_status st = check_ws(ws, ws_bytes, L.total);
    if (st != SPECDEC_OK) return st;
    Pass1Params P;
    fill_common(P, logits, row_stride, V_shard, L, rows, 1, 1, ws);
    P.vocab_offset = vocab_offset;
    P.shard_keys = row_keys;
    P.shard_vals = row_vals;
    P.topk = topk;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (topk > 0) return dispatch_shard_rows<MODE_TOP8>(dtype, vec, P, s);
    return dispatch_shard_rows<MODE_ARGMAX>(dtype, vec, P, s);
}

specdec_status specdec_shard_greedy_combine(const uint64_t* gathered_keys, const float* gathered_vals, int world,
                                            const int32_t* draft_tokens, int B, int k, int V, int32_t* accept_len,
                                            int32_t* out_tokens, int topk, int32_t* topk_ids, float* topk_vals,
                                            struct CUstream_st* stream) {
    if (world < 1 || world > 32 || B < 0 || B > SPECDEC_MAX_B || k < 0 || k > SPECDEC_MAX_K || V < 1 ||
        V > SPECDEC_MAX_V || topk < 0 || topk > SPECDEC_MAX_TOPK)
        return SPECDEC_ERR_INVALID_ARG;
    if (B == 0) return SPECDEC_OK;
    if (gathered_keys == nullptr || accept_len == nullptr || out_tokens == nullptr) return SPECDEC_ERR_INVALID_ARG;
    if (k > 0 && draft_tokens == nullptr) return SPECDEC_ERR_INVALID_ARG;
    if (topk > 0 && (gathered_vals == nullptr || topk_ids == nullptr || topk_vals == nullptr))
        return SPECDEC_ERR_INVALID_ARG;
    Pass1Params P;
    memset(&P, 0, sizeof(P));
    P.V = V;
    P.R = static_cast<int64_t>(B) * (k + 1);
    P.B = B;
    P.k = k;
    P.drafts = draft_tokens;
    P.accept_len = accept_len;
    P.out_tokens = out_tokens;
    P.topk = topk;
    P.topk_ids = topk_ids;
    P.topk_vals = topk_vals;
    P.gathered_keys = gathered_keys;
    P.gathered_vals = gathered_vals;
    P.world = world;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = topk > 0 ? launch_pdl(verify_shard_combine_kernel<MODE_TOP8>, dim3(static_cast<unsigned>(B)), 0, s, P)
                             : launch_pdl(verify_shard_combine_kernel<MODE_ARGMAX>, dim3(static_cast<unsigned>(B)), 0, s, P);
    if (e != cudaSuccess) return SPECDEC_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? SPECDEC_OK : SPECDEC_ERR_CUDA;
}

size_t specdec_workspace_size_shard_rejection(int B, int k, int V_shard, specdec_dtype dtype) {
    if (!dtype_ok(dtype) || B < 0 || B > SPECDEC_MAX_B || k < 0 || k > SPECDEC_MAX_K || V_shard < 1 ||
        V_shard > SPECDEC_MAX_V)
        return 0;
    const Layout a = shard_rej_layout(B, k, V_shard, vec_elems(dtype));
    const Layout b = shard_rej_layout(B, k, V_shard, 1);
    return a.total > b.total ? a.total : b.total;
}

specdec_status specdec_shard_rejection_rows(const void* target, specdec_dtype dtype, int64_t row_stride,
                                            const float* draft_probs, int64_t q_row_stride,
                                            const int32_t* draft_tokens, int B, int k, int V_shard, int vocab_offset,
                                            float temperature, void* row_stats, void* ws, size_t ws_bytes,
                                            struct CUstream_st* stream) {
    if (!dtype_ok(dtype)) return SPECDEC_ERR_UNSUPPORTED;
    if (B < 0 || B > SPECDEC_MAX_B || k < 0 || k > SPECDEC_MAX_K || V_shard < 1 || V_shard > SPECDEC_MAX_V ||
        vocab_offset < 0 || static_cast<int64_t>(vocab_offset) + V_shard > SPECDEC_MAX_V)
        return SPECDEC_ERR_INVALID_ARG;
    if (!(isnormal(temperature) && temperature > 0.0f)) return SPECDEC_ERR_INVALID_ARG;
    if (B == 0) return SPECDEC_OK;
    const int64_t rows = static_cast<int64_t>(B) * (k + 1);
    if (!rows_fit(rows, row_stride, V_shard)) return SPECDEC_ERR_INVALID_ARG;
    if (target == nullptr || row_stats == nullptr) return SPECDEC_ERR_INVALID_ARG;
    if (k > 0 && (draft_tokens == nullptr || draft_probs == nullptr ||
                  !rows_fit(static_cast<int64_t>(B) * k, q_row_stride, V_shard)))
        return SPECDEC_ERR_INVALID_ARG;
    const bool vec = vector_path_ok(target, row_stride, elem_size(dtype)) &&
                     (k == 0 || vector_path_ok(draft_probs, q_row_stride, 4));
    const Layout L = shard_rej_layout(B, k, V_shard, vec ? vec_elems(dtype) : 1);
    specdec_status st = check_ws(ws, ws_bytes, L.total);
    if (st != SPECDEC_OK) return st;
    const double invT_d = 1.0 / static_cast<double>(temperature);
    Pass1Params P;
    fill_common(P, target, row_stride, V_shard, L, rows, k + 1, B, ws);
    P.drafts = draft_tokens;
    P.k = k;
    P.q = draft_probs;
    P.q_stride = q_row_stride;
    P.invT = static_cast<float>(invT_d);
    P.log2e_invT = static_cast<float>(invT_d * 1.4426950408889634);
    P.invT_d = invT_d;
    P.vocab_offset = vocab_offset;
    P.shard_stats = static_cast<ShardRowStat*>(row_stats);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (P.R > 0x7fffffff || P.cpr > 65535) return SPECDEC_ERR_UNSUPPORTED;
    const dim3 grid(static_cast<unsigned>(P.R), static_cast<unsigned>(P.cpr));
    const dim3 grid2(static_cast<unsigned>((P.R + NWARPS - 1) / NWARPS));
    cudaError_t e;
    if (dtype == SPECDEC_BF16) {
        e = vec ? launch_pdl(verify_pass1_kernel<BF16Tag, 8, MODE_SOFTMAX>, grid, 0, s, P)
                : launch_pdl(verify_pass1_kernel<BF16Tag, 1, MODE_SOFTMAX>, grid, 0, s, P);
        if (e == cudaSuccess) e = launch_pdl(verify_shard_softmax_rows_kernel<BF16Tag>, grid2, 0, s, P);
    } else {
        e = vec ? launch_pdl(verify_pass1_kernel<F32Tag, 4, MODE_SOFTMAX>, grid, 0, s, P)
                : launch_pdl(verify_pass1_kernel<F32Tag, 1, MODE_SOFTMAX>, grid, 0, s, P);
        if (e == cudaSuccess) e = launch_pdl(verify_shard_softmax_rows_kernel<F32Tag>, grid2, 0, s, P);
    }
    if (e != cudaSuccess) return SPECDEC_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? SPECDEC_OK : SPECDEC_ERR_CUDA;
}

specdec_status specdec_shard_rejection_decide(const void* gathered_row_stats, int world, const int32_t* draft_tokens,
                                              int B, int k, int V, float temperature, uint64_t seed, uint64_t offset,
                                              int32_t* accept_len, int32_t* out_tokens, float* p_draft_out,
                                              void* ws, size_t ws_bytes, struct CUstream_st* stream) {
    if (world < 1 || world > 32 || B < 0 || B > SPECDEC_MAX_B || k < 0 || k > SPECDEC_MAX_K || V < 1 ||
        V > SPECDEC_MAX_V)
        return SPECDEC_ERR_INVALID_ARG;
    if (!(isnormal(temperature) && temperature > 0.0f)) return SPECDEC_ERR_INVALID_ARG;
    if (B == 0) return SPECDEC_OK;
    if (gathered_row_stats == nullptr || accept_len == nullptr || out_tokens == nullptr) return SPECDEC_ERR_INVALID_ARG;
    if (k > 0 && draft_tokens == nullptr) return SPECDEC_ERR_INVALID_ARG;
    specdec_status st = check_ws(ws, ws_bytes, kPartialBase + static_cast<size_t>(B) * sizeof(RejState));
    if (st != SPECDEC_OK) return st;
    const double invT_d = 1.0 / static_cast<double>(temperature);
    Pass1Params P;
    memset(&P, 0, sizeof(P));
    P.V = V;
    P.R = static_cast<int64_t>(B) * (k + 1);
    P.B = B;
    P.k = k;
    P.drafts = draft_tokens;
    P.accept_len = accept_len;
    P.out_tokens = out_tokens;
    P.p_draft_out = p_draft_out;
    P.invT_d = invT_d;
    P.seed = seed;
    P.offset = offset;
    P.world = world;
    P.gathered_stats = static_cast<const ShardRowStat*>(gathered_row_stats);
    P.state = reinterpret_cast<RejState*>(static_cast<char*>(ws) + kPartialBase);
    if (launch_pdl(verify_shard_decide_kernel, dim3(static_cast<unsigned>(B)), 0, reinterpret_cast<cudaStream_t>(stream),
                   P) != cudaSuccess)
        return SPECDEC_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? SPECDEC_OK : SPECDEC_ERR_CUDA;
}

namespace {
// Pass-2 parameters of a shard-rejection step (masses or token search).
Pass2Params shard_pass2_params(const void* target, int64_t row_stride, const float* q, int64_t q_stride, int B,
                               int k, int V_shard, float temperature, uint64_t seed, uint64_t offset, const Layout& L,
                               void* ws) {
    Pass2Params Q;
    memset(&Q, 0, sizeof(Q));
    const double invT_d = 1.0 / static_cast<double>(temperature);
    Q.logits = target;
    Q.row_stride = row_stride;
    Q.q = q;
    Q.q_stride = q_stride;
    Q.V = V_shard;
    Q.nv_full = static_cast<int>(L.nv_full);
    Q.cpr = static_cast<int>(L.cpr2);
    Q.B = B;
    Q.k = k;
    Q.invT = static_cast<float>(invT_d);
    Q.log2e_invT = static_cast<float>(invT_d * 1.4426950408889634);
    Q.seed = seed;
    Q.offset = offset;
    Q.state = reinterpret_cast<RejState*>(static_cast<char*>(ws) + L.state);
    Q.chunk_mass = reinterpret_cast<double2*>(static_cast<char*>(ws) + L.masses);
    Q.unit_mass = reinterpret_cast<double2*>(static_cast<char*>(ws) + L.units);
    return Q;
}
}  // namespace

specdec_status specdec_shard_rejection_masses(const void* target, specdec_dtype dtype, int64_t row_stride,
                                              const float* draft_probs, int64_t q_row_stride, int B, int k,
                                              int V_shard, float temperature, double* masses, void* ws,
                                              size_t ws_bytes, struct CUstream_st* stream) {
    if (!dtype_ok(dtype)) return SPECDEC_ERR_UNSUPPORTED;
    if (B < 0 || B > SPECDEC_MAX_B || k < 0 || k > SPECDEC_MAX_K || V_shard < 1 || V_shard > SPECDEC_MAX_V)
        return SPECDEC_ERR_INVALID_ARG;
    if (!(isnormal(temperature) && temperature > 0.0f)) return SPECDEC_ERR_INVALID_ARG;
    if (B == 0) return SPECDEC_OK;
    if (target == nullptr || masses == nullptr || (k > 0 && draft_probs == nullptr)) return SPECDEC_ERR_INVALID_ARG;
    const bool vec = vector_path_ok(target, row_stride, elem_size(dtype)) &&
                     (k == 0 || vector_path_ok(draft_probs, q_row_stride, 4));
    const Layout L = shard_rej_layout(B, k, V_shard, vec ? vec_elems(dtype) : 1);
    specdec_status st = check_ws(ws, ws_bytes, L.total);
    if (st != SPECDEC_OK) return st;
    Pass2Params Q = shard_pass2_params(target, row_stride, draft_probs, q_row_stride, B, k, V_shard, temperature, 0,
                                       0, L, ws);
    Q.shard_mass_out = reinterpret_cast<double2*>(masses);
    if (Q.cpr > 65535) return SPECDEC_ERR_UNSUPPORTED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const dim3 grid(static_cast<unsigned>(B), static_cast<unsigned>(Q.cpr));
    const dim3 grid2(static_cast<unsigned>((B + NWARPS - 1) / NWARPS));
    cudaError_t e;
    if (dtype == SPECDEC_BF16)
        e = vec ? launch_pdl(verify_resample_kernel<BF16Tag, 8>, grid, 0, s, Q)
                : launch_pdl(verify_resample_kernel<BF16Tag, 1>, grid, 0, s, Q);
    else
        e = vec ? launch_pdl(verify_resample_kernel<F32Tag, 4>, grid, 0, s, Q)
                : launch_pdl(verify_resample_kernel<F32Tag, 1>, grid, 0, s, Q);
    if (e == cudaSuccess)
        e = launch_pdl(verify_shard_mass_totals_kernel, grid2, 0, s, Q);
    if (e != cudaSuccess) return SPECDEC_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? SPECDEC_OK : SPECDEC_ERR_CUDA;
}

specdec_status specdec_shard_rejection_sample(const void* target, specdec_dtype dtype, int64_t row_stride,
                                              const float* draft_probs, int64_t q_row_stride, int B, int k,
                                              int V_shard, int vocab_offset, float temperature, uint64_t seed,
                                              uint64_t offset, const double* gathered_masses, int world, int rank,
                                              int32_t* shard_tokens, void* ws, size_t ws_bytes,
                                              struct CUstream_st* stream) {
    if (!dtype_ok(dtype)) return SPECDEC_ERR_UNSUPPORTED;
    if (B < 0 || B > SPECDEC_MAX_B || k < 0 || k > SPECDEC_MAX_K || V_shard < 1 || V_shard > SPECDEC_MAX_V ||
        world < 1 || world > 32 || rank < 0 || rank >= world || vocab_offset < 0 ||
        static_cast<int64_t>(vocab_offset) + V_shard > SPECDEC_MAX_V)
        return SPECDEC_ERR_INVALID_ARG;
    if (!(isnormal(temperature) && temperature > 0.0f)) return SPECDEC_ERR_INVALID_ARG;
    if (B == 0) return SPECDEC_OK;
    if (target == nullptr || gathered_masses == nullptr || shard_tokens == nullptr) return SPECDEC_ERR_INVALID_ARG;
    const bool vec = vector_path_ok(target, row_stride, elem_size(dtype)) &&
                     (k == 0 || vector_path_ok(draft_probs, q_row_stride, 4));
    const Layout L = shard_rej_layout(B, k, V_shard, vec ? vec_elems(dtype) : 1);
    specdec_status st = check_ws(ws, ws_bytes, L.total);
    if (st != SPECDEC_OK) return st;
    Pass2Params Q = shard_pass2_params(target, row_stride, draft_probs, q_row_stride, B, k, V_shard, temperature,
                                       seed, offset, L, ws);
    Q.shard_totals = reinterpret_cast<const double2*>(gathered_masses);
    Q.world = world;
    Q.rank = rank;
    Q.vocab_offset = vocab_offset;
    Q.shard_token = shard_tokens;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const dim3 grid(static_cast<unsigned>((B + NWARPS - 1) / NWARPS));
    cudaError_t e;
    if (dtype == SPECDEC_BF16)
        e = vec ? launch_pdl(verify_resample_epilogue_kernel<BF16Tag, 8>, grid, 0, s, Q)
                : launch_pdl(verify_resample_epilogue_kernel<BF16Tag, 1>, grid, 0, s, Q);
    else
        e = vec ? launch_pdl(verify_resample_epilogue_kernel<F32Tag, 4>, grid, 0, s, Q)
                : launch_pdl(verify_resample_epilogue_kernel<F32Tag, 1>, grid, 0, s, Q);
    if (e != cudaSuccess) return SPECDEC_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? SPECDEC_OK : SPECDEC_ERR_CUDA;
}

specdec_status specdec_shard_rejection_finish(const int32_t* gathered_tokens, int world, int B, int k,
                                              int32_t* out_tokens, void* ws, size_t ws_bytes,
                                              struct CUstream_st* stream) {
    if (world < 1 || world > 32 || B < 0 || B > SPECDEC_MAX_B || k < 0 || k > SPECDEC_MAX_K)
        return SPECDEC_ERR_INVALID_ARG;
    if (B == 0) return SPECDEC_OK;
    if (gathered_tokens == nullptr || out_tokens == nullptr) return SPECDEC_ERR_INVALID_ARG;
    specdec_status st = check_ws(ws, ws_bytes, kPartialBase + static_cast<size_t>(B) * sizeof(RejState));
    if (st != SPECDEC_OK) return st;
    Pass1Params P;
    memset(&P, 0, sizeof(P));
    P.B = B;
    P.k = k;
    P.out_tokens = out_tokens;
    P.world = world;
    P.gathered_tokens = gathered_tokens;
    P.state = reinterpret_cast<RejState*>(static_cast<char*>(ws) + kPartialBase);
    if (launch_pdl(verify_shard_finish_kernel, dim3(static_cast<unsigned>((B + NT - 1) / NT)), 0,
                   reinterpret_cast<cudaStream_t>(stream), P) != cudaSuccess)
        return SPECDEC_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? SPECDEC_OK : SPECDEC_ERR_CUDA;
}

size_t specdec_workspace_size_ragged(specdec_mode mode, int B, int total_drafts, int V, specdec_dtype dtype) {
    if (!dtype_ok(dtype) || B < 0 || B > SPECDEC_MAX_B || V < 1 || V > SPECDEC_MAX_V) return 0;
    if (mode != SPECDEC_MODE_GREEDY && mode != SPECDEC_MODE_REJECTION) return 0;
    if (total_drafts < 0 || static_cast<int64_t>(total_drafts) > static_cast<int64_t>(B) * SPECDEC_MAX_K) return 0;
    const int64_t rows = static_cast<int64_t>(B) + total_drafts;
    const bool rej = mode == SPECDEC_MODE_REJECTION;
    const Layout a = make_layout(rows, 1, B, V, vec_elems(dtype), slot_bytes(mode), rej);
    const Layout b = make_layout(rows, 1, B, V, 1, slot_bytes(mode), rej);
    return a.total > b.total ? a.total : b.total;
}

specdec_status specdec_workspace_init(void* ws, size_t bytes, struct CUstream_st* stream) {
    if (ws == nullptr || reinterpret_cast<uintptr_t>(ws) % 16 != 0) return SPECDEC_ERR_WORKSPACE;
    if (bytes == 0) return SPECDEC_OK;
    return cudaMemsetAsync(ws, 0, bytes, stream) == cudaSuccess ? SPECDEC_OK : SPECDEC_ERR_CUDA;
}

specdec_status specdec_verify_greedy(const void* logits, specdec_dtype dtype, int64_t row_stride,
                                     const int32_t* draft_tokens, int B, int k, int V,
                                     int32_t* accept_len, int32_t* out_tokens,
                                     int topk, int32_t* topk_ids, float* topk_vals,
                                     void* ws, size_t ws_bytes, struct CUstream_st* stream) {
    const specdec_status st = greedy_args_status(logits, dtype, row_stride, draft_tokens, B, k, V, accept_len,
                                                 out_tokens, topk, topk_ids, topk_vals);
    if (st != SPECDEC_OK || B == 0) return st;
    return greedy_impl(logits, dtype, row_stride, draft_tokens, nullptr, static_cast<int64_t>(B) * k, B, k, V,
                       accept_len, out_tokens, topk, topk_ids, topk_vals, nullptr, ws, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

specdec_status specdec_verify_greedy_ragged(const void* logits, specdec_dtype dtype, int64_t row_stride,
                                            const int32_t* draft_tokens, const int32_t* draft_offsets, int B,
                                            int total_drafts, int max_k, int V, int32_t* accept_len,
                                            int32_t* out_tokens, int topk, int32_t* topk_ids, float* topk_vals,
                                            int64_t* counters, void* ws, size_t ws_bytes,
                                            struct CUstream_st* stream) {
    if (!dtype_ok(dtype)) return SPECDEC_ERR_UNSUPPORTED;
    if (B < 0 || B > SPECDEC_MAX_B || V < 1 || V > SPECDEC_MAX_V) return SPECDEC_ERR_INVALID_ARG;
    if (topk < 0 || topk > SPECDEC_MAX_TOPK) return SPECDEC_ERR_INVALID_ARG;
    if (!ragged_args_ok(draft_offsets, B, total_drafts, max_k)) return SPECDEC_ERR_INVALID_ARG;
    if (B == 0) return SPECDEC_OK;
    return greedy_impl(logits, dtype, row_stride, draft_tokens, draft_offsets, total_drafts, B, max_k, V, accept_len,
                       out_tokens, topk, topk_ids, topk_vals, counters, ws, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

specdec_status specdec_verify_tree(const void* logits, specdec_dtype dtype, int64_t row_stride,
                                   const int32_t* parents, const int32_t* node_tokens,
                                   int B, int N, int V, int max_depth,
                                   int32_t* accept_len, int32_t* accept_nodes, int32_t* out_tokens,
                                   void* ws, size_t ws_bytes, struct CUstream_st* stream) {
    if (!dtype_ok(dtype)) return SPECDEC_ERR_UNSUPPORTED;
    if (B < 0 || B > SPECDEC_MAX_B || N < 0 || N + 1 > SPECDEC_MAX_TREE_NODES || V < 1 || V > SPECDEC_MAX_V)
        return SPECDEC_ERR_INVALID_ARG;
    if (max_depth < 1 || max_depth > SPECDEC_MAX_DEPTH) return SPECDEC_ERR_INVALID_ARG;
    if (B == 0) return SPECDEC_OK;
    const int64_t rows = static_cast<int64_t>(B) * (N + 1);
    if (!rows_fit(rows, row_stride, V)) return SPECDEC_ERR_INVALID_ARG;
    if (logits == nullptr || parents == nullptr || node_tokens == nullptr || accept_len == nullptr ||
        accept_nodes == nullptr || out_tokens == nullptr)
        return SPECDEC_ERR_INVALID_ARG;
    const bool vec = vector_path_ok(logits, row_stride, elem_size(dtype));
    const int ve = vec ? vec_elems(dtype) : 1;
    const Layout L = make_layout(rows, N + 1, B, V, ve, kArgmaxChunkBytes, false);
    specdec_status st = check_ws(ws, ws_bytes, L.total);
    if (st != SPECDEC_OK) return st;
    Pass1Params P;
    fill_common(P, logits, row_stride, V, L, rows, N + 1, B, ws);
    P.parents = parents;
    P.node_tokens = node_tokens;
    P.max_depth = max_depth;
    P.accept_len = accept_len;
    P.accept_nodes = accept_nodes;
    P.out_tokens = out_tokens;
    return dispatch_pass1<MODE_TREE>(dtype, vec, P, reinterpret_cast<cudaStream_t>(stream));
}

specdec_status specdec_verify_rejection(const void* target_logits, specdec_dtype dtype, int64_t row_stride,
                                        const float* draft_probs, int64_t q_row_stride,
                                        const int32_t* draft_tokens, int B, int k, int V,
                                        float temperature, uint64_t seed, uint64_t offset,
                                        int32_t* accept_len, int32_t* out_tokens, float* p_draft_out,
                                        void* ws, size_t ws_bytes, struct CUstream_st* stream) {
    if (!dtype_ok(dtype)) return SPECDEC_ERR_UNSUPPORTED;
    if (B < 0 || B > SPECDEC_MAX_B || k < 0 || k > SPECDEC_MAX_K || V < 1 || V > SPECDEC_MAX_V)
        return SPECDEC_ERR_INVALID_ARG;
    if (!(isnormal(temperature) && temperature > 0.0f)) return SPECDEC_ERR_INVALID_ARG;
    if (B == 0) return SPECDEC_OK;
    return rejection_impl(target_logits, dtype, row_stride, draft_probs, q_row_stride, draft_tokens, nullptr,
                          static_cast<int64_t>(B) * k, B, k, V, temperature, seed, offset, accept_len, out_tokens,
                          p_draft_out, nullptr, nullptr, nullptr, ws, ws_bytes,
                          reinterpret_cast<cudaStream_t>(stream));
}

specdec_status specdec_verify_rejection_slice(const void* target_logits, specdec_dtype dtype, int64_t row_stride,
                                              const float* draft_probs, int64_t q_row_stride,
                                              const int32_t* draft_tokens, int B, int k, int V, float temperature,
                                              uint64_t seed, uint64_t offset, uint32_t request_base,
                                              int32_t* accept_len, int32_t* out_tokens, float* p_draft_out,
                                              void* ws, size_t ws_bytes, struct CUstream_st* stream) {
    if (!dtype_ok(dtype)) return SPECDEC_ERR_UNSUPPORTED;
    if (B < 0 || B > SPECDEC_MAX_B || k < 0 || k > SPECDEC_MAX_K || V < 1 || V > SPECDEC_MAX_V)
        return SPECDEC_ERR_INVALID_ARG;
    if (!(isnormal(temperature) && temperature > 0.0f)) return SPECDEC_ERR_INVALID_ARG;
    if (static_cast<uint64_t>(request_base) + static_cast<uint64_t>(B) > (uint64_t(1) << 32))
        return SPECDEC_ERR_INVALID_ARG;  // a request index past 2^32 - 1
    if (B == 0) return SPECDEC_OK;
    return rejection_impl(target_logits, dtype, row_stride, draft_probs, q_row_stride, draft_tokens, nullptr,
                          static_cast<int64_t>(B) * k, B, k, V, temperature, seed, offset, accept_len, out_tokens,
                          p_draft_out, nullptr, nullptr, nullptr, ws, ws_bytes,
                          reinterpret_cast<cudaStream_t>(stream), request_base);
}

specdec_status specdec_verify_rejection_stats(const void* target_logits, specdec_dtype dtype, int64_t row_stride,
                                              const float* draft_probs, int64_t q_row_stride,
                                              const int32_t* draft_tokens, int B, int k, int V, float temperature,
                                              uint64_t seed, uint64_t offset, int32_t* accept_len,
                                              int32_t* out_tokens, float* p_draft_out, double* draft_entropy,
                                              double* js_distance, void* ws, size_t ws_bytes,
                                              struct CUstream_st* stream) {
    if (!dtype_ok(dtype)) return SPECDEC_ERR_UNSUPPORTED;
    if (B < 0 || B > SPECDEC_MAX_B || k < 0 || k > SPECDEC_MAX_K || V < 1 || V > SPECDEC_MAX_V)
        return SPECDEC_ERR_INVALID_ARG;
    if (!(isnormal(temperature) && temperature > 0.0f)) return SPECDEC_ERR_INVALID_ARG;
    if (k > 0 && (draft_entropy == nullptr || js_distance == nullptr)) return SPECDEC_ERR_INVALID_ARG;
    if (B == 0) return SPECDEC_OK;
    return rejection_impl(target_logits, dtype, row_stride, draft_probs, q_row_stride, draft_tokens, nullptr,
                          static_cast<int64_t>(B) * k, B, k, V, temperature, seed, offset, accept_len, out_tokens,
                          p_draft_out, nullptr, draft_entropy, js_distance, ws, ws_bytes,
                          reinterpret_cast<cudaStream_t>(stream));
}

specdec_status specdec_verify_rejection_ragged(const void* target_logits, specdec_dtype dtype, int64_t row_stride,
                                               const float* draft_probs, int64_t q_row_stride,
                                               const int32_t* draft_tokens, const int32_t* draft_offsets, int B,
                                               int total_drafts, int max_k, int V, float temperature, uint64_t seed,
                                               uint64_t offset, int32_t* accept_len, int32_t* out_tokens,
                                               float* p_draft_out, int64_t* counters, void* ws, size_t ws_bytes,
                                               struct CUstream_st* stream) {
    if (!dtype_ok(dtype)) return SPECDEC_ERR_UNSUPPORTED;
    if (B < 0 || B > SPECDEC_MAX_B || V < 1 || V > SPECDEC_MAX_V) return SPECDEC_ERR_INVALID_ARG;
    if (!(isnormal(temperature) && temperature > 0.0f)) return SPECDEC_ERR_INVALID_ARG;
    if (!ragged_args_ok(draft_offsets, B, total_drafts, max_k)) return SPECDEC_ERR_INVALID_ARG;
    if (B == 0) return SPECDEC_OK;
    return rejection_impl(target_logits, dtype, row_stride, draft_probs, q_row_stride, draft_tokens, draft_offsets,
                          total_drafts, B, max_k, V, temperature, seed, offset, accept_len, out_tokens, p_draft_out,
                          counters, nullptr, nullptr, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

specdec_status specdec_ngram_propose(const int32_t* tokens, int64_t token_stride, const int32_t* lengths, int B,
                                     int n_min, int n_max, int k, int32_t* drafts, int32_t* num_drafts,
                                     int32_t* draft_offsets, int32_t* packed_drafts, struct CUstream_st* stream) {
    if (B < 0 || B > SPECDEC_MAX_B || n_min < 1 || n_max < n_min || n_max > kNgramMax || k < 0 ||
        k > SPECDEC_MAX_K || token_stride < 1 || token_stride > (int64_t(1) << 31) - 1)
        return SPECDEC_ERR_INVALID_ARG;
    if ((draft_offsets == nullptr) != (packed_drafts == nullptr)) return SPECDEC_ERR_INVALID_ARG;
    if (B == 0) return SPECDEC_OK;
    if (tokens == nullptr || lengths == nullptr || num_drafts == nullptr || (k > 0 && drafts == nullptr))
        return SPECDEC_ERR_INVALID_ARG;
    NgramParams P;
    P.tokens = tokens;
    P.stride = token_stride;
    P.lengths = lengths;
    P.B = B;
    P.n_min = n_min;
    P.n_max = n_max;
    P.k = k;
    P.drafts = drafts;
    P.num_drafts = num_drafts;
    P.offsets = draft_offsets;
    P.packed = packed_drafts;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (launch_pdl(verify_ngram_kernel, dim3(static_cast<unsigned>(B)), 0, s, P) != cudaSuccess) return SPECDEC_ERR_CUDA;
    if (draft_offsets != nullptr && launch_pdl(verify_ngram_pack_kernel, dim3(1), 0, s, P) != cudaSuccess)
        return SPECDEC_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? SPECDEC_OK : SPECDEC_ERR_CUDA;
}

int specdec_set_prefetch_inputs(int enable) { return g_prefetch_inputs.exchange(enable ? 1 : 0); }

double specdec_tier_update(specdec_tier_state* state, double accepted, double decay) {
    if (state == nullptr || !(decay >= 0.0 && decay < 1.0) || !(accepted >= 0.0 && accepted <= SPECDEC_MAX_K))
        return NAN;
    if (!state->initialized) {
        state->ema = accepted;
        state->initialized = 1;
    } else {
        state->ema = decay * state->ema + (1.0 - decay) * accepted;
    }
    return state->ema;
}

int specdec_tier_select(const int* tiers, int n_tiers, double ema) {
    if (tiers == nullptr || n_tiers < 1 || !(ema >= 0.0)) return -1;
    for (int i = 0; i < n_tiers; ++i) {
        if (tiers[i] < 0 || tiers[i] > SPECDEC_MAX_K) return -1;
        if (i > 0 && tiers[i] <= tiers[i - 1]) return -1;
    }
    for (int i = 0; i < n_tiers; ++i)
        if (static_cast<double>(tiers[i]) >= ema + 0.5) return tiers[i];
    return tiers[n_tiers - 1];
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Greedy verification with library-owned scratch (no allocation anywhere).
//
// Some callers cannot allocate device memory: plug-ins and engine hooks that
// are handed only their input and output pointers and no allocator, or code
// running in a process whose memory pool already owns the whole GPU (a
// serving engine that reserved HBM for its KV cache up front), where a
// cudaMalloc would fail or fragment the pool.  For them the scratch lives in
// a fixed file-scope device array of SPECDEC_STATIC_SCRATCH_BYTES, which
// every GPU that loads this library holds until the process exits.
//
// Host code must not pass `g_static_scratch` itself to a kernel: on the host
// that name is only a stand-in for the device symbol.  The device address is
// looked up once per device with cudaGetSymbolAddress, with that device
// current, on the first call made on it.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_static_scratch[SPECDEC_STATIC_SCRATCH_BYTES];

namespace specdec {
namespace {
std::atomic<void*> g_static_scratch_addr[kMaxDevices];

// Device address of this device's copy of g_static_scratch (set-up on the
// first call per device; later calls read the cached pointer).
cudaError_t static_scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    void* p = g_static_scratch_addr[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return e;
        g_static_scratch_addr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return cudaSuccess;
}
}  // namespace
}  // namespace specdec

extern "C" specdec_status specdec_verify_greedy_static_scratch(
    const void* logits, specdec_dtype dtype, int64_t row_stride, const int32_t* draft_tokens, int B, int k, int V,
    int32_t* accept_len, int32_t* out_tokens, int topk, int32_t* topk_ids, float* topk_vals,
    struct CUstream_st* stream) {
    // Every argument check comes before the first CUDA call, so a rejected
    // call enqueues nothing (not even the threshold clear below).
    specdec_status st = specdec::greedy_args_status(logits, dtype, row_stride, draft_tokens, B, k, V, accept_len,
                                                    out_tokens, topk, topk_ids, topk_vals);
    if (st != SPECDEC_OK || B == 0) return st;
    const size_t need = specdec_workspace_size(SPECDEC_MODE_GREEDY, B, k, V, dtype);
    if (need > SPECDEC_STATIC_SCRATCH_BYTES) return SPECDEC_ERR_WORKSPACE;  // beyond the fixed scratch
    void* scratch = nullptr;
    if (specdec::static_scratch_address(&scratch) != cudaSuccess) return SPECDEC_ERR_CUDA;
    // The top-8 row thresholds must start at zero.  Every completed call
    // leaves them so, but the array keeps whatever a call that failed
    // half-way left: clear this call's words first.
    if (topk > 0) {
        int64_t rows = static_cast<int64_t>(B) * (k + 1);
        if (rows > specdec::kThetaRows) rows = specdec::kThetaRows;
        if (cudaMemsetAsync(static_cast<char*>(scratch) + specdec::kThetaBase, 0,
                            static_cast<size_t>(rows) * sizeof(unsigned),
                            reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
            return SPECDEC_ERR_CUDA;
    }
    return specdec_verify_greedy(logits, dtype, row_stride, draft_tokens, B, k, V, accept_len, out_tokens, topk,
                                 topk_ids, topk_vals, scratch, SPECDEC_STATIC_SCRATCH_BYTES, stream);
}
