// Whole-model decode step: every layer's append and decode attention recorded once into a
// CUDA graph and replayed per generated token.  Host-side only: the recorded work is the
// library's own entry points (kvq_quantize_append, kvq_decode_attention or its fused form),
// so a replay runs exactly the kernels, arguments and order of those calls.
#include <new>

#include "kvq_common.cuh"

using namespace kvq_host;

struct kvq_step {
    cudaGraphExec_t exec;
    void* inputs;       // the graph's input record (device)
    size_t input_bytes;
};

namespace {

constexpr int kMaxStepLayers = 4096;

// Byte sizes of one layer's parts of the packed input record.
struct StepParts {
    size_t kv;  // k (and v): fp16 [B][n_new][Hkv][D]
    size_t q;   // q: fp16 [B][Hq][D]
    size_t layer() const { return 2 * kv + q; }
};

StepParts step_parts(const kvq_cfg* cfg, int32_t n_new) {
    StepParts p;
    p.kv = (size_t)cfg->B * n_new * cfg->Hkv * cfg->D * 2;
    p.q = (size_t)cfg->B * cfg->Hq * cfg->D * 2;
    return p;
}

size_t pad16(size_t x) { return (x + 15) & ~(size_t)15; }

int attention_ws(const kvq_cfg* cfg, int32_t max_len, int32_t splits, int32_t fused,
                 size_t* bytes) {
    return fused ? kvq_decode_fused_workspace(cfg, max_len, splits, bytes)
                 : kvq_decode_workspace(cfg, max_len, splits, bytes);
}

}  // namespace

extern "C" {

int kvq_step_input_bytes(const kvq_cfg* cfg, int32_t layers, int32_t n_new, size_t* bytes) {
    int e = check_cfg(cfg);
    if (e) return e;
    if (!bytes) return KVQ_ERR_NULL;
    if (layers < 1 || layers > kMaxStepLayers || n_new < 0 || n_new > cfg->T_max)
        return KVQ_ERR_SHAPE;
    *bytes = (size_t)layers * step_parts(cfg, n_new).layer() + pad16((size_t)cfg->B * 4);
    return KVQ_OK;
}

int kvq_step_workspace(const kvq_cfg* cfg, int32_t n_new, int32_t max_len, int32_t splits,
                       int32_t fused, size_t* bytes) {
    int e = check_cfg(cfg);
    if (e) return e;
    if (!bytes) return KVQ_ERR_NULL;
    if (n_new < 0 || n_new > cfg->T_max || (fused != 0 && fused != 1)) return KVQ_ERR_SHAPE;
    size_t aws = 0, dws = 0;
    if (n_new > 0 && (e = kvq_quantize_workspace(cfg, n_new, 0, &aws))) return e;
    if ((e = attention_ws(cfg, max_len, splits, fused, &dws))) return e;
    *bytes = align_up(aws) + dws;
    return KVQ_OK;
}

int kvq_step_create(const kvq_cfg* cfg, const kvq_step_desc* d, kvq_step** step) {
    if (!step) return KVQ_ERR_NULL;
    *step = nullptr;
    int e = check_cfg(cfg);
    if (e) return e;
    if (!d || !d->caches || !d->cbK || !d->cbV || !d->inputs || !d->out || !d->workspace)
        return KVQ_ERR_NULL;
    if (!aligned16(d->inputs) || !aligned16(d->out) || !aligned16(d->workspace))
        return KVQ_ERR_ALIGN;
    size_t in_bytes = 0, ws_bytes = 0, aws = 0;
    if ((e = kvq_step_input_bytes(cfg, d->layers, d->n_new, &in_bytes))) return e;
    if ((e = kvq_step_workspace(cfg, d->n_new, d->max_len, d->splits, d->fused, &ws_bytes)))
        return e;
    if (d->workspace_bytes < ws_bytes) return KVQ_ERR_WORKSPACE;
    if (d->n_new > 0 && (e = kvq_quantize_workspace(cfg, d->n_new, 0, &aws))) return e;
    const StepParts P = step_parts(cfg, d->n_new);
    uint8_t* in = static_cast<uint8_t*>(d->inputs);
    const int32_t* qpos = reinterpret_cast<const int32_t*>(in + (size_t)d->layers * P.layer());
    uint8_t* app_ws = static_cast<uint8_t*>(d->workspace);
    uint8_t* att_ws = app_ws + align_up(aws);
    const size_t att_bytes = d->workspace_bytes - align_up(aws);
    const size_t out_stride = (size_t)cfg->B * cfg->Hq * cfg->D;

    cudaStream_t cs = nullptr;
    cudaError_t ce = cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking);
    if (ce) return record_cuda(ce);
    ce = cudaStreamBeginCapture(cs, cudaStreamCaptureModeRelaxed);
    if (ce) {
        cudaStreamDestroy(cs);
        return record_cuda(ce);
    }
    for (int32_t l = 0; l < d->layers && !e; ++l) {
        const uint8_t* base = in + (size_t)l * P.layer();
        const uint16_t* k = reinterpret_cast<const uint16_t*>(base);
        const uint16_t* v = reinterpret_cast<const uint16_t*>(base + P.kv);
        const uint16_t* q = reinterpret_cast<const uint16_t*>(base + 2 * P.kv);
        if (d->n_new > 0)
            e = kvq_quantize_append(cfg, &d->caches[l], &d->cbK[l], &d->cbV[l], k, v, d->n_new,
                                    nullptr, 0, app_ws, aws, cs);
        if (e) break;
        float* out = d->out + (size_t)l * out_stride;
        e = d->fused ? kvq_decode_attention_fused(cfg, &d->caches[l], &d->cbK[l], &d->cbV[l], q,
                                                  qpos, d->max_len, out, att_ws, att_bytes,
                                                  d->splits, cs)
                     : kvq_decode_attention(cfg, &d->caches[l], &d->cbK[l], &d->cbV[l], q, qpos,
                                            d->max_len, out, att_ws, att_bytes, d->splits, cs);
    }
    cudaGraph_t graph = nullptr;
    ce = cudaStreamEndCapture(cs, &graph);  // always ends the capture, also after an error
    if (!e && ce) e = record_cuda(ce);
    cudaGraphExec_t exec = nullptr;
    if (!e) {
        ce = cudaGraphInstantiate(&exec, graph, 0);
        if (ce) e = record_cuda(ce);
    }
    if (graph) cudaGraphDestroy(graph);  // the instantiated graph keeps what it needs
    cudaStreamDestroy(cs);
    if (e) {
        if (exec) cudaGraphExecDestroy(exec);
        return e;
    }
    kvq_step* s = new (std::nothrow) kvq_step{exec, d->inputs, in_bytes};
    if (!s) {
        cudaGraphExecDestroy(exec);
        return record_cuda(cudaErrorMemoryAllocation);
    }
    *step = s;
    return KVQ_OK;
}

int kvq_step_launch(kvq_step* s, const void* inputs, void* stream) {
    if (!s) return KVQ_ERR_NULL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (inputs) {
        cudaError_t ce = cudaMemcpyAsync(s->inputs, inputs, s->input_bytes, cudaMemcpyDefault, st);
        if (ce) return record_cuda(ce);
    }
    return record_cuda(cudaGraphLaunch(s->exec, st));
}

int kvq_step_destroy(kvq_step* s) {
    if (!s) return KVQ_ERR_NULL;
    cudaError_t ce = cudaGraphExecDestroy(s->exec);
    delete s;
    return record_cuda(ce);
}

}  // extern "C"
