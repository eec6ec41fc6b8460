// Host-side entry points of libkvq that hold no method arithmetic: configuration
// checks, array sizes, cache reset, status read-back and error strings.
#include <stdio.h>
#include <string.h>

#include "kvq_common.cuh"

namespace kvq_host {

static thread_local char g_cuda_msg[256] = "no CUDA error recorded";

int record_cuda(cudaError_t e) {
    if (e == cudaSuccess) return KVQ_OK;
    snprintf(g_cuda_msg, sizeof(g_cuda_msg), "CUDA error %d: %s", (int)e, cudaGetErrorString(e));
    return KVQ_ERR_CUDA;
}

int check_cfg(const kvq_cfg* cfg) {
    if (!cfg) return KVQ_ERR_NULL;
    if (cfg->D != kvq::kD) return KVQ_ERR_UNSUPPORTED;
    if (cfg->bits < 2 || cfg->bits > 4) return KVQ_ERR_UNSUPPORTED;
    if (cfg->B < 1 || cfg->B > 65535) return KVQ_ERR_SHAPE;
    if (cfg->Hkv < 1 || cfg->Hkv > 64) return KVQ_ERR_SHAPE;
    if (cfg->Hq < cfg->Hkv || cfg->Hq % cfg->Hkv != 0 || cfg->Hq / cfg->Hkv > 16) return KVQ_ERR_SHAPE;
    if (cfg->T_max < 1 || cfg->T_max > (1 << 24)) return KVQ_ERR_SHAPE;
    if (cfg->out_cap_k < 0 || cfg->out_cap_v < 0) return KVQ_ERR_SHAPE;
    if ((cfg->out_cap_k | cfg->out_cap_v) & 7) return KVQ_ERR_SHAPE;  // lists stay 16-byte aligned
    if (!(cfg->outlier_frac >= 0.0 && cfg->outlier_frac <= 1.0)) return KVQ_ERR_SHAPE;
    if (!(cfg->rope_theta > 1.0)) return KVQ_ERR_SHAPE;
    return KVQ_OK;
}

int check_cache(const kvq_cfg* cfg, const kvq_cache* c) {
    if (!c) return KVQ_ERR_NULL;
    const void* ptrs[] = {c->kcodes, c->vcodes, c->kthr, c->kparams, c->vparams, c->kchunk,
                          c->vchunk, c->kcount, c->vcount, c->len, c->status};
    for (const void* p : ptrs) {
        if (!p) return KVQ_ERR_NULL;
        if (!aligned16(p)) return KVQ_ERR_ALIGN;
    }
    if (cfg->out_cap_k > 0 && !c->kout) return KVQ_ERR_NULL;
    if (cfg->out_cap_v > 0 && !c->vout) return KVQ_ERR_NULL;
    const void* opt[] = {c->kout, c->vout};
    for (const void* p : opt)
        if (p && !aligned16(p)) return KVQ_ERR_ALIGN;
    return KVQ_OK;
}

int check_codebook(const kvq_codebook* cb) {
    if (!cb || !cb->levels || !cb->bounds) return KVQ_ERR_NULL;
    return KVQ_OK;
}

size_t align_up(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace kvq_host

using namespace kvq_host;

extern "C" {

int kvq_abi_version(void) { return KVQ_ABI_VERSION; }

const char* kvq_strerror(int code) {
    switch (code) {
        case KVQ_OK: return "ok";
        case KVQ_ERR_NULL: return "a required pointer is NULL";
        case KVQ_ERR_ALIGN: return "a device pointer is not 16-byte aligned";
        case KVQ_ERR_SHAPE: return "a dimension or count is out of range";
        case KVQ_ERR_UNSUPPORTED: return "unsupported bits or head_dim (need D=128, bits 2..4)";
        case KVQ_ERR_RANGE: return "token range or split count out of range";
        case KVQ_ERR_WORKSPACE: return "workspace too small";
        case KVQ_ERR_CUDA: return g_cuda_msg;
        case KVQ_ERR_SCRATCH_LIMIT:
            return "request needs more scratch than the fixed no-alloc array holds";
        default: return "unknown kvq error code";
    }
}

int kvq_validate_cfg(const kvq_cfg* cfg) { return check_cfg(cfg); }

int kvq_layout(const kvq_cfg* cfg, kvq_sizes* out) {
    int e = check_cfg(cfg);
    if (e) return e;
    if (!out) return KVQ_ERR_NULL;
    const size_t B = cfg->B, T = cfg->T_max, n = (size_t)cfg->Hkv * cfg->D;
    const size_t nch = kvq::nchunks(cfg->T_max) + 1;
    out->kcodes = B * (size_t)kvq::nquads(cfg->T_max) * cfg->Hkv * kvq::block_words(cfg->bits) * 4;
    out->vcodes = out->kcodes;
    out->kthr = B * n * 2 * 2;
    out->kparams = B * n * 2 * 4;
    out->vparams = B * T * 2 * 4;
    const size_t BH = B * (size_t)cfg->Hkv;  // one outlier list per (sequence, kv head)
    out->kout = BH * cfg->out_cap_k * 4;
    out->vout = BH * cfg->out_cap_v * 4;
    out->kchunk = BH * nch * 4;
    out->vchunk = BH * nch * 4;
    out->kcount = BH * 4;
    out->vcount = BH * 4;
    out->len = B * 4;
    out->status = 4;
    return KVQ_OK;
}

int kvq_cache_reset(const kvq_cfg* cfg, const kvq_cache* c, void* stream) {
    int e = check_cfg(cfg);
    if (e) return e;
    if ((e = check_cache(cfg, c))) return e;
    kvq_sizes sz;
    kvq_layout(cfg, &sz);
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t ce;
    if ((ce = cudaMemsetAsync(c->kchunk, 0, sz.kchunk, st))) return record_cuda(ce);
    if ((ce = cudaMemsetAsync(c->vchunk, 0, sz.vchunk, st))) return record_cuda(ce);
    if ((ce = cudaMemsetAsync(c->kcount, 0, sz.kcount, st))) return record_cuda(ce);
    if ((ce = cudaMemsetAsync(c->vcount, 0, sz.vcount, st))) return record_cuda(ce);
    if ((ce = cudaMemsetAsync(c->len, 0, sz.len, st))) return record_cuda(ce);
    if ((ce = cudaMemsetAsync(c->status, 0, sz.status, st))) return record_cuda(ce);
    return KVQ_OK;
}

int kvq_get_status(const kvq_cache* c, int32_t* out, void* stream) {
    if (!c || !c->status || !out) return KVQ_ERR_NULL;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t ce = cudaMemcpyAsync(out, c->status, 4, cudaMemcpyDeviceToHost, st);
    if (ce) return record_cuda(ce);
    return record_cuda(cudaStreamSynchronize(st));
}

}  // extern "C"
