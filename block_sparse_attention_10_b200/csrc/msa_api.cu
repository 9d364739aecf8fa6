// msa_api.cu — the C ABI of libmsa.so (see include/msa.h): host-side argument
// checks, then the kernel launches.  No allocation, no host synchronisation.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "internal.h"

namespace msa {

const DeviceInfo& device_info() {
    static thread_local DeviceInfo cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    DeviceInfo& di = cache[dev];
    if (di.device != dev) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) == cudaSuccess) {
            di.num_sms = prop.multiProcessorCount;
            di.smem_optin = prop.sharedMemPerBlockOptin;
        } else {
            di.num_sms = 148;
            di.smem_optin = 227 * 1024;
        }
        di.device = dev;
    }
    return di;
}

namespace {

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

bool good_scale(float s) { return std::isfinite(s) && s > 0.0f; }

int check_cache(const msa_nvfp4_cache_t& c) {
    if (!c.data || !c.scale) return MSA_EINVAL;
    if (!good_scale(c.tensor_scale)) return MSA_EINVAL;
    if (!aligned16(c.data) || !aligned16(c.scale)) return MSA_EALIGN;
    return MSA_OK;
}

bool is_pow2_le8(int x) { return x == 1 || x == 2 || x == 4 || x == 8; }

// Checks shared by the MSA steps; `need_*` selects which inputs the step reads.
int check_params(const msa_params_t* p, bool need_index, bool need_attend) {
    if (!p) return MSA_EINVAL;
    if (p->B <= 0 || p->Tq <= 0 || p->lmax <= 0 || !p->seq_lens) return MSA_EINVAL;
    if (p->lmax % MSA_BLOCK_TOKENS != 0) return MSA_EINVAL;
    if (p->lmax > (int64_t(1) << 31)) return MSA_EUNSUPPORTED;
    if (p->Tq > p->lmax) return MSA_EINVAL;
    if (p->pool_mode != 0 && p->pool_mode != 1) return MSA_EINVAL;
    if (p->block_table != nullptr && p->num_pages <= 0) return MSA_EINVAL;
    if (p->out_bf16 != 0 && p->out_bf16 != 1) return MSA_EINVAL;
    if (need_index) {
        if (p->HI <= 0 || p->DI <= 0 || !p->q_idx) return MSA_EINVAL;
        if (int r = check_cache(p->ik)) return r;
        if (!aligned16(p->q_idx)) return MSA_EALIGN;
        if (p->DI != 64 && p->DI != 128) return MSA_EUNSUPPORTED;
        if (!is_pow2_le8(p->HI)) return MSA_EUNSUPPORTED;
        if ((int64_t)p->Tq * p->HI > 32 && p->pool_mode != 0) return MSA_EUNSUPPORTED;  // prefill: mean only
        if (p->B > 4096) return MSA_EUNSUPPORTED;
    }
    if (need_attend) {
        if (p->Hq <= 0 || p->Hkv <= 0 || p->D <= 0 || !p->q) return MSA_EINVAL;
        if (p->Hq % p->Hkv != 0) return MSA_EINVAL;
        if (int r = check_cache(p->k)) return r;
        if (int r = check_cache(p->v)) return r;
        if (!aligned16(p->q)) return MSA_EALIGN;
        if (p->D != 128) return MSA_EUNSUPPORTED;
        if (!is_pow2_le8(p->Hq / p->Hkv)) return MSA_EUNSUPPORTED;
        if (!(std::isfinite(p->softmax_scale) && p->softmax_scale >= 0.0f)) return MSA_EINVAL;
    }
    return MSA_OK;
}

Problem to_problem(const msa_params_t* p) {
    Problem q;
    q.B = p->B;
    q.Tq = p->Tq;
    q.Hq = p->Hq;
    q.Hkv = p->Hkv;
    q.D = p->D;
    q.HI = p->HI;
    q.DI = p->DI;
    q.lmax = p->lmax;
    q.nbmax = p->lmax / MSA_BLOCK_TOKENS;
    q.seq_lens = p->seq_lens;
    q.k = Cache{p->k.data, p->k.scale, p->k.tensor_scale};
    q.v = Cache{p->v.data, p->v.scale, p->v.tensor_scale};
    q.ik = Cache{p->ik.data, p->ik.scale, p->ik.tensor_scale};
    q.q = static_cast<const __nv_bfloat16*>(p->q);
    q.q_idx = static_cast<const __nv_bfloat16*>(p->q_idx);
    q.w_idx = p->w_idx;
    q.softmax_scale = p->softmax_scale > 0.0f ? p->softmax_scale : 1.0f / sqrtf((float)p->D);
    q.pool_mode = p->pool_mode;
    q.status = p->status;
    q.block_table = p->block_table;
    q.num_pages = p->block_table != nullptr ? p->num_pages : 0;
    q.out_bf16 = p->out_bf16;
    q.blk_lo = 0;
    q.blk_hi = q.nbmax;
    return q;
}

// Programmatic dependent launch between the decode kernels (on unless MSA_PDL=0).
bool pdl_enabled() {
    static const bool on = [] {
        const char* e = std::getenv("MSA_PDL");
        return !(e != nullptr && e[0] == '0');
    }();
    return on;
}

}  // namespace

// Decode indexer (mma.sync, Tq * HI <= 32) or prefill indexer (tcgen05, larger Tq * HI).
int launch_index(const Problem& p, float* block_scores, float* token_scores, bool pdl, cudaStream_t st) {
    if ((int64_t)p.Tq * p.HI <= 32) return launch_index_decode(p, block_scores, token_scores, pdl, st);
    if (token_scores != nullptr) return MSA_EUNSUPPORTED;
    return launch_index_prefill(p, block_scores, pdl, st);
}

namespace {

constexpr size_t kAlign = 256;
size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

size_t ws_block_scores_bytes(const msa_params_t* p) {
    return round_up((size_t)p->B * p->Tq * (size_t)(p->lmax / MSA_BLOCK_TOKENS) * sizeof(float));
}
size_t ws_sel_bytes(const msa_params_t* p) {
    return round_up((size_t)p->B * p->Tq * MSA_TOPK_BLOCKS * sizeof(int32_t));
}

}  // namespace
}  // namespace msa

using namespace msa;

extern "C" {

const char* msa_status_string(int code) {
    switch (code) {
        case MSA_OK: return "MSA_OK";
        case MSA_EINVAL: return "MSA_EINVAL: invalid argument";
        case MSA_EUNSUPPORTED: return "MSA_EUNSUPPORTED: shape not supported by the kernels";
        case MSA_EALIGN: return "MSA_EALIGN: pointer not 16-byte aligned";
        case MSA_EWORKSPACE: return "MSA_EWORKSPACE: workspace missing, misaligned or too small";
        case MSA_ECUDA: return "MSA_ECUDA: CUDA launch error";
        default: return "MSA: unknown status";
    }
}

const char* msa_version(void) { return "libmsa 0.1 (sm_100a)"; }

int msa_nvfp4_encode(const float* x, int64_t nvec, int dim, float tensor_scale, uint8_t* data, uint8_t* scale,
                     cudaStream_t stream) {
    if (nvec < 0 || dim <= 0 || dim % 16 != 0) return MSA_EINVAL;
    if (nvec == 0) return MSA_OK;
    if (!x || !data || !scale || !good_scale(tensor_scale)) return MSA_EINVAL;
    if (!aligned16(x) || !aligned16(data)) return MSA_EALIGN;
    return launch_nvfp4_encode(x, nvec, dim, tensor_scale, data, scale, stream);
}

int msa_nvfp4_decode(const uint8_t* data, const uint8_t* scale, int64_t nvec, int dim, float tensor_scale,
                     float* out, cudaStream_t stream) {
    if (nvec < 0 || dim <= 0 || dim % 16 != 0) return MSA_EINVAL;
    if (nvec == 0) return MSA_OK;
    if (!out || !data || !scale || !good_scale(tensor_scale)) return MSA_EINVAL;
    if (!aligned16(out) || !aligned16(data)) return MSA_EALIGN;
    return launch_nvfp4_decode(data, scale, nvec, dim, tensor_scale, out, stream);
}

int msa_nvfp4_amax(const float* x, int64_t n, float* amax_out, cudaStream_t stream) {
    if (n < 0 || !amax_out || (n > 0 && !x)) return MSA_EINVAL;
    return launch_nvfp4_amax(x, n, amax_out, stream);
}

size_t msa_workspace_size(const msa_params_t* p) {
    if (check_params(p, true, true) != MSA_OK) return 0;
    return ws_block_scores_bytes(p) + ws_sel_bytes(p) + attend_prefill_ws_bytes(to_problem(p));
}

size_t msa_workspace_size_single_launch(const msa_params_t* p) {
    if (check_params(p, true, true) != MSA_OK) return 0;
    const Problem q = to_problem(p);
    return fused_supported(q) ? fused_layout(q).total : 0;
}

int msa_index(const msa_params_t* p, float* block_scores, float* token_scores, cudaStream_t stream) {
    if (int r = check_params(p, true, false)) return r;
    if (!block_scores) return MSA_EINVAL;
    return launch_index(to_problem(p), block_scores, token_scores, false, stream);
}

int msa_select(const msa_params_t* p, const float* block_scores, int32_t* sel, cudaStream_t stream) {
    if (int r = check_params(p, false, false)) return r;
    if (!block_scores || !sel) return MSA_EINVAL;
    return launch_select(to_problem(p), block_scores, sel, nullptr, false, stream);
}

int msa_attend(const msa_params_t* p, const int32_t* sel, void* out_, float* lse, cudaStream_t stream) {
    float* out = static_cast<float*>(out_);  // bf16 elements when out_bf16
    if (int r = check_params(p, false, true)) return r;
    if (!sel || !out) return MSA_EINVAL;
    if (!aligned16(out)) return MSA_EALIGN;
    return launch_attend(to_problem(p), sel, out, lse, false, stream);
}

int msa_decode(const msa_params_t* p, void* ws, size_t ws_bytes, void* out_, float* lse, int32_t* sel_out,
               cudaStream_t stream) {
    float* out = static_cast<float*>(out_);  // bf16 elements when out_bf16
    if (int r = check_params(p, true, true)) return r;
    if (!out) return MSA_EINVAL;
    if (!aligned16(out)) return MSA_EALIGN;
    const Problem q = to_problem(p);
    const size_t need = ws_block_scores_bytes(p) + ws_sel_bytes(p) + attend_prefill_ws_bytes(q);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return MSA_EWORKSPACE;
    float* bs = static_cast<float*>(ws);
    int32_t* sel = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + ws_block_scores_bytes(p));
    const bool pdl = pdl_enabled();
    if (int r = launch_index(q, bs, nullptr, pdl, stream)) return r;
    // chunked prefill: block-major tensor-core attention over the inverted selection
    if (attend_prefill_supported(q)) {
        if (int r = launch_select(q, bs, sel, sel_out, pdl, stream)) return r;
        void* ws_ap = static_cast<uint8_t*>(ws) + ws_block_scores_bytes(p) + ws_sel_bytes(p);
        return launch_attend_prefill(q, sel, ws_ap, out, lse, pdl, stream);
    }
    // short rows: each attention CTA selects its own row's blocks (one launch fewer)
    if (q.nbmax <= 1024) return launch_select_attend(q, bs, sel_out, out, lse, pdl, stream);
    if (int r = launch_select(q, bs, sel, sel_out, pdl, stream)) return r;
    return launch_attend(q, sel, out, lse, pdl, stream);
}

int msa_decode_single_launch(const msa_params_t* p, void* ws, size_t ws_bytes, void* out_, float* lse,
                             int32_t* sel_out, cudaStream_t stream) {
    float* out = static_cast<float*>(out_);  // bf16 elements when out_bf16
    if (int r = check_params(p, true, true)) return r;
    if (!out) return MSA_EINVAL;
    if (!aligned16(out)) return MSA_EALIGN;
    const Problem q = to_problem(p);
    if (!fused_supported(q)) return MSA_EUNSUPPORTED;
    if (!ws || ws_bytes < fused_layout(q).total || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0)
        return MSA_EWORKSPACE;
    return launch_decode_fused(q, ws, out, lse, sel_out, pdl_enabled(), stream);
}

// ---------------------------------------------------------------- context-parallel decode

size_t msa_dcp_workspace_size(const msa_params_t* p) {
    if (check_params(p, true, false) != MSA_OK) return 0;
    return ws_block_scores_bytes(p);
}

int msa_dcp_candidates(const msa_params_t* p, int64_t n0, int64_t n1, void* ws, size_t ws_bytes,
                       float* cand_score, int32_t* cand_id, cudaStream_t stream) {
    if (int r = check_params(p, true, false)) return r;
    if (!cand_score || !cand_id) return MSA_EINVAL;
    Problem q = to_problem(p);
    if (n0 < 0 || n1 <= n0 || n1 > q.nbmax) return MSA_EINVAL;
    if ((int64_t)p->Tq * p->HI > 32) return MSA_EUNSUPPORTED;  // decode indexer only
    if (!ws || ws_bytes < ws_block_scores_bytes(p) || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0)
        return MSA_EWORKSPACE;
    q.blk_lo = n0;
    q.blk_hi = n1;
    float* bs = static_cast<float*>(ws);
    const bool pdl = pdl_enabled();
    if (int r = launch_index_decode(q, bs, nullptr, pdl, stream)) return r;
    return launch_dcp_candidates(q, bs, cand_score, cand_id, pdl, stream);
}

int msa_dcp_merge(const msa_params_t* p, int G, const float* cand_score, const int32_t* cand_id, int32_t* sel,
                  cudaStream_t stream) {
    if (int r = check_params(p, false, false)) return r;
    if (!cand_score || !cand_id || !sel) return MSA_EINVAL;
    if (G < 1) return MSA_EINVAL;
    if (G > kDcpMaxRanks) return MSA_EUNSUPPORTED;
    return launch_dcp_merge(to_problem(p), G, cand_score, cand_id, sel, false, stream);
}

int msa_dcp_attend(const msa_params_t* p, int64_t n0, int64_t n1, const int32_t* sel, float* out, float* lse,
                   cudaStream_t stream) {
    if (int r = check_params(p, false, true)) return r;
    if (!sel || !out || !lse) return MSA_EINVAL;
    if (!aligned16(out)) return MSA_EALIGN;
    Problem q = to_problem(p);
    if (n0 < 0 || n1 <= n0 || n1 > q.nbmax) return MSA_EINVAL;
    q.blk_lo = n0;
    q.blk_hi = n1;
    q.out_bf16 = 0;  // partials stay fp32 until the combine
    return launch_attend(q, sel, out, lse, false, stream);
}

int msa_dcp_combine(const msa_params_t* p, int G, const float* part_out, const float* part_lse, void* out_,
                    float* lse, cudaStream_t stream) {
    float* out = static_cast<float*>(out_);  // bf16 elements when out_bf16
    if (int r = check_params(p, false, true)) return r;
    if (!part_out || !part_lse || !out) return MSA_EINVAL;
    if (!aligned16(part_out) || !aligned16(out)) return MSA_EALIGN;
    if (G < 1) return MSA_EINVAL;
    if (G > kDcpMaxRanks) return MSA_EUNSUPPORTED;
    return launch_dcp_combine(to_problem(p), G, part_out, part_lse, out, lse, false, stream);
}

}  // extern "C"
