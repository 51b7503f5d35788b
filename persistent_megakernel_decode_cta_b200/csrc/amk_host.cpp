// amk_host.cpp -- the C ABI of libamk (declared in include/amk.h): handle
// lifetime, device memory, the per-token cooperative launch and error
// reporting.
//
// "RightNow-AI/AutoMegaKernel" README, opening summary and "What is built and
// verified": one launch per token, a KV cache carried across steps, and an
// unsafe schedule rejected at validation instead of hanging the GPU
// ("Deadlock-free by construction").
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <algorithm>
#include <atomic>
#include <cstring>
#include <new>
#include <vector>

#include "amk.h"
#include "amk_internal.h"
#include "amk_plan.h"

using amk::ErrorWord;
using amk::KParams;
using amk::TaskDesc;

extern "C" cudaError_t amk_kernel_configure(int smem_bytes, int quant, int att_e, int generic,
                                            int fused);
extern "C" cudaError_t amk_pack_down(const void *wd, void *out, int h, int ffn, int esz,
                                     cudaStream_t stream);
extern "C" cudaError_t amk_pack_q4(const void *codes, const void *scales, void *out, int rows,
                                   int K, cudaStream_t stream);
extern "C" cudaError_t amk_kernel_occupancy(int smem_bytes, int quant, int att_e, int generic,
                                            int fused, int *blocks_per_sm);
namespace amk {
extern "C" cudaError_t amk_kernel_launch(const KParams *p, int n_ctas, int smem_bytes,
                                         cudaStream_t stream);
}

namespace {
thread_local char g_last_error[512] = "";
}

extern "C" int amk_set_error(int code, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return code;
}

extern "C" const char *amk_last_error(void) { return g_last_error; }

extern "C" const char *amk_version(void) { return "amk-b200 0.1 (sm_100a)"; }

extern "C" const char *amk_strerror(int s)
{
    switch (s) {
    case AMK_OK: return "ok";
    case AMK_ERR_INVALID_ARG: return "invalid argument";
    case AMK_ERR_UNSUPPORTED: return "unsupported shape";
    case AMK_ERR_VALIDATION: return "schedule rejected by the validator";
    case AMK_ERR_POS_RANGE: return "position or token out of range";
    case AMK_ERR_LAUNCH: return "cooperative launch refused";
    case AMK_ERR_TIMEOUT: return "device wait timed out";
    case AMK_ERR_CUDA: return "CUDA runtime error";
    case AMK_ERR_OOM: return "device allocation failed";
    case AMK_ERR_POISONED: return "handle poisoned by an earlier timeout; call amk_reset_kv";
    case AMK_ERR_NO_DEVICE: return "no CUDA device";
    default: return "unknown status";
    }
}

extern "C" int amk_default_options(amk_options *o)
{
    if (!o)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_default_options: NULL");
    memset(o, 0, sizeof *o);
    o->ring_stages = 0;  // ring shape resolved by the lowering from the weight format
    o->stage_bytes = 0;
    o->attn_splits = 0;
    o->tasks_per_sm = 1;
    o->n_sms = 0;
    o->wait_timeout_us = 1000000;  // 1 s
    o->debug_skip_signal_task = -1;
    o->ffn_fused = 1;
    o->pos0_plan = 1;
    o->flagged_waits = 1;
    return AMK_OK;
}

// ---------------------------------------------------------------- host plans
extern "C" int amk_plan_create(const amk_config *cfg, const amk_options *opt, int32_t n_sms,
                               amk_plan **out, amk_validation_report *report)
{
    if (!cfg || !out)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_plan_create: NULL argument");
    *out = nullptr;
    static std::atomic<uint64_t> next_uid{1};
    amk_plan *P = new (std::nothrow) amk_plan();
    if (!P)
        return amk_set_error(AMK_ERR_OOM, "amk_plan_create: out of host memory");
    P->uid = next_uid.fetch_add(1);
    auto lower_checked = [&](amk_plan *Q, int pos0) {
        int r = amk_lower(cfg, opt, n_sms, Q, pos0);
        if (r == AMK_OK) {
            amk_graph g;
            amk_plan_view(Q, &g);
            amk_validation_report local;
            r = amk_validate_graph(&g, report ? report : &local);
            if (r != AMK_OK)
                amk_set_error(r, "lowered %sschedule rejected: %s", pos0 ? "position-0 " : "",
                              (report ? report : &local)->message);
        }
        return r;
    };
    int rc = lower_checked(P, 0);
    if (rc == AMK_OK && P->opt.pos0_plan > 0) {
        P->pos0 = new (std::nothrow) amk_plan();
        if (P->pos0)
            P->pos0->uid = next_uid.fetch_add(1);
        rc = P->pos0 ? lower_checked(P->pos0, 1)
                     : amk_set_error(AMK_ERR_OOM, "amk_plan_create: out of host memory");
    }
    if (rc != AMK_OK) {
        delete P;
        return rc;
    }
    *out = P;
    return AMK_OK;
}

extern "C" const amk_plan *amk_plan_pos0(const amk_plan *p) { return p ? p->pos0 : nullptr; }

extern "C" int amk_plan_graph(const amk_plan *p, amk_graph *out)
{
    if (!p || !out)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_plan_graph: NULL argument");
    amk_plan_view(p, out);
    return AMK_OK;
}

extern "C" int amk_plan_task_info(const amk_plan *p, int32_t *kind, int32_t *layer)
{
    if (!p)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_plan_task_info: NULL plan");
    const size_t n = p->tasks.size();
    if (kind)
        memcpy(kind, p->kind.data(), n * sizeof(int32_t));
    if (layer)
        memcpy(layer, p->layer.data(), n * sizeof(int32_t));
    return AMK_OK;
}

extern "C" void amk_plan_destroy(amk_plan *p) { delete p; }

// ---------------------------------------------------------------- handles
struct amk_handle {
    amk_plan *plan = nullptr;
    int device = 0;
    cudaStream_t stream = nullptr;
    std::vector<void *> dev_allocs;
    // debug_checks: a guard of kGuardBytes after every device buffer the handle
    // owns, filled with kGuardByte at create
    bool guards_on = false;
    std::vector<const void *> guards;
    TaskDesc *d_tasks = nullptr;
    int32_t *d_qoff = nullptr;
    uint32_t *d_ctr = nullptr;
    // the position-0 schedule (plan->pos0): its own tables and level counters
    TaskDesc *d_tasks0 = nullptr;
    int32_t *d_qoff0 = nullptr;
    uint32_t *d_ctr0 = nullptr;
    uint32_t epoch0 = 0;  // steps run with it since the last reset
    ErrorWord *d_err = nullptr;
    uint64_t *d_qkv = nullptr, *d_attn = nullptr, *d_xmid = nullptr,
             *d_xout = nullptr;  // flagged words
    uint32_t *d_act = nullptr;  // 32-bit flagged words
    float *d_part = nullptr, *d_logits = nullptr;
    uint32_t tag = 0;  // tag of the last step's flagged words (0: none yet)
    unsigned long long *d_argkey = nullptr;
    long long *d_xacc = nullptr;    // [L][h] fixed-point residual (fused FFN)
    void *d_act_block = nullptr;    // every activation buffer, one allocation
    void *d_dpack = nullptr;        // [L] packed Wdown (fused FFN), see KParams::dpack
    void *d_q4 = nullptr;           // W4A16: every int4 matrix as rows of codes + scales
    unsigned long long *d_prof = nullptr;
    uint16_t *d_kv = nullptr;
    size_t kv_bytes = 0, act_bytes = 0, fw_bytes = 0;  // fw: the flagged words from d_qkv
    ErrorWord *h_err = nullptr;            // pinned
    unsigned long long *h_key = nullptr;   // pinned
    cudaEvent_t err_ev = nullptr;
    bool err_pending = false;
    KParams kp{};
    uint32_t epoch = 0;
    uint32_t arrive_base = 0;  // attention chunk arrivals so far, per (layer, kv head)
    bool poisoned = false;
    amk_error_info last_err{};
};

namespace {

int cuda_fail(cudaError_t e, const char *what)
{
    return amk_set_error(e == cudaErrorMemoryAllocation ? AMK_ERR_OOM : AMK_ERR_CUDA, "%s: %s",
                         what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return p && ((uintptr_t)p % 16) == 0; }

constexpr size_t kGuardBytes = 256;
constexpr int kGuardByte = 0xA5;

template <typename T>
int dalloc(amk_handle *H, T **out, size_t bytes)
{
    void *p = nullptr;
    bytes = bytes ? bytes : 16;
    const size_t body = (bytes + 15) & ~(size_t)15;
    cudaError_t e = cudaMalloc(&p, H->guards_on ? body + kGuardBytes : bytes);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaMalloc");
    H->dev_allocs.push_back(p);
    if (H->guards_on) {
        uint8_t *g = static_cast<uint8_t *>(p) + body;
        if ((e = cudaMemset(g, kGuardByte, kGuardBytes)) != cudaSuccess)
            return cuda_fail(e, "guard fill");
        H->guards.push_back(g);
    }
    *out = static_cast<T *>(p);
    return AMK_OK;
}

// Debug bounds check of resolved task records (amk_options.debug_checks):
// every GEMV tile's rows lie within its matrix, its chunk geometry covers
// them, and every attention tile's KV blocks lie within the handle's cache.
int check_task_records(const amk_plan *P, const std::vector<TaskDesc> &ts, const uint16_t *kv,
                       size_t kv_bytes)
{
    const amk_config &c = P->cfg;
    const int hq = c.n_heads * c.head_dim, hk = c.n_kv_heads * c.head_dim;
    for (size_t i = 0; i < ts.size(); ++i) {
        const TaskDesc &d = ts[i];
        auto bad = [&](const char *what) {
            return amk_set_error(AMK_ERR_VALIDATION, "debug check: task %zu (kind %d, layer %d): %s",
                                 i, d.kind, d.layer, what);
        };
        if (d.layer < 0 || d.layer >= c.n_layers)
            return bad("layer out of range");
        if (d.kind == amk::TK_ATTN) {
            const uint8_t *lo = reinterpret_cast<const uint8_t *>(kv);
            const size_t blk = (size_t)c.max_ctx * c.head_dim * 2;
            for (const void *w : {d.w0, d.w1}) {
                const uint8_t *q = static_cast<const uint8_t *>(w);
                if (q < lo || q + blk > lo + kv_bytes)
                    return bad("KV block outside the cache");
            }
            if (d.r0 < 0 || d.r0 >= c.n_kv_heads || d.r1 < 0 || d.r1 >= P->opt.attn_splits)
                return bad("attention head or chunk out of range");
            continue;
        }
        int rows = c.hidden;
        switch (d.kind) {
        case amk::TK_QKV: rows = d.mat == 0 ? hq : hk; break;
        case amk::TK_GATEUP: case amk::TK_FFN: rows = c.ffn; break;
        case amk::TK_LMHEAD: rows = c.vocab; break;
        default: break;  // OPROJ, DOWN: hidden rows
        }
        const int R = d.r1 - d.r0;
        if (d.r0 < 0 || R <= 0 || d.r1 > rows || R > amk::kMaxTaskRows)
            return bad("row range outside the matrix or above the task limit");
        if (!d.w0 || d.rpc == 0 || d.nck == 0 || (int)d.nck * d.rpc < R ||
            ((int)d.nck - 1) * d.rpc >= R)
            return bad("chunk geometry does not cover the rows exactly");
        const int parts = (d.kind == amk::TK_GATEUP || d.kind == amk::TK_FFN) ? 2 : 1;
        if (d.ngu != d.nck * parts ||
            d.nchunks != d.ngu + (d.kind == amk::TK_FFN ? d.nck2 : 0) ||
            (1 << d.ks_log2) * (1 << d.rg_log2) != amk::kConsumerWarps || d.rpc % (1 << d.rg_log2))
            return bad("chunk or warp geometry inconsistent");
        if (d.kind == amk::TK_FFN && ((int)d.nck2 * d.rpc2 < c.hidden || d.ncb == 0))
            return bad("fused FFN Wdown chunks do not cover hidden");
    }
    return AMK_OK;
}

void free_handle(amk_handle *H)
{
    if (!H)
        return;
    if (H->stream)
        cudaStreamSynchronize(H->stream);
    for (void *p : H->dev_allocs)
        cudaFree(p);
    if (H->h_err)
        cudaFreeHost(H->h_err);
    if (H->h_key)
        cudaFreeHost(H->h_key);
    if (H->err_ev)
        cudaEventDestroy(H->err_ev);
    delete H->plan;
    delete H;
}

int check_weights(const amk_config *c, const amk_weights *w)
{
    if (!aligned16(w->embed) || !aligned16(w->final_norm))
        return amk_set_error(AMK_ERR_INVALID_ARG, "embed/final_norm NULL or not 16-byte aligned");
    if (!c->tied_embeddings) {
        if (!aligned16(w->lm_head))
            return amk_set_error(AMK_ERR_INVALID_ARG, "lm_head NULL or not 16-byte aligned");
        if (c->quant != AMK_QUANT_BF16 && !w->lm_head_scale)
            return amk_set_error(AMK_ERR_INVALID_ARG, "lm_head_scale NULL for int8/int4 weights");
    }
    const void *const *mats[7] = {w->wq, w->wk, w->wv, w->wo, w->wgate, w->wup, w->wdown};
    const void *const *scs[7] = {w->sq, w->sk, w->sv, w->so, w->sgate, w->sup, w->sdown};
    if (!w->attn_norm || !w->ffn_norm)
        return amk_set_error(AMK_ERR_INVALID_ARG, "norm pointer arrays NULL");
    for (int m = 0; m < 7; ++m) {
        if (!mats[m])
            return amk_set_error(AMK_ERR_INVALID_ARG, "weight pointer array %d NULL", m);
        if (c->quant != AMK_QUANT_BF16 && !scs[m])
            return amk_set_error(AMK_ERR_INVALID_ARG, "scale pointer array %d NULL", m);
    }
    for (int l = 0; l < c->n_layers; ++l) {
        if (!aligned16(w->attn_norm[l]) || !aligned16(w->ffn_norm[l]))
            return amk_set_error(AMK_ERR_INVALID_ARG, "layer %d norm NULL or misaligned", l);
        for (int m = 0; m < 7; ++m) {
            if (!aligned16(mats[m][l]))
                return amk_set_error(AMK_ERR_INVALID_ARG, "layer %d weight %d NULL or not "
                                     "16-byte aligned", l, m);
            if (c->quant != AMK_QUANT_BF16 && !scs[m][l])
                return amk_set_error(AMK_ERR_INVALID_ARG, "layer %d scale %d NULL", l, m);
        }
    }
    return AMK_OK;
}

int zero_state(amk_handle *H)
{
    const amk_plan *P = H->plan;
    cudaError_t e;
    e = cudaMemsetAsync(H->d_kv, 0, H->kv_bytes, H->stream);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(H->d_ctr, 0, sizeof(uint32_t) * (size_t)(P->n_counters + P->n_arrive),
                            H->stream);
    if (e == cudaSuccess && P->pos0)
        e = cudaMemsetAsync(H->d_ctr0, 0, sizeof(uint32_t) * (size_t)P->pos0->n_counters,
                            H->stream);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(H->d_err, 0, sizeof(ErrorWord), H->stream);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(H->d_argkey, 0, 2 * sizeof(unsigned long long), H->stream);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(H->d_act_block, 0, H->act_bytes, H->stream);
    if (e != cudaSuccess)
        return cuda_fail(e, "amk_reset_kv");
    H->epoch = 0;
    H->epoch0 = 0;
    H->tag = 0;  // the flagged words were cleared with the block above
    H->arrive_base = 0;
    H->poisoned = false;
    H->err_pending = false;
    memset(&H->last_err, 0, sizeof H->last_err);
    return AMK_OK;
}

// Maps a device error word to a status; poisons the handle on failure.
int absorb_error(amk_handle *H, const ErrorWord &e)
{
    if (e.code == 0)
        return AMK_OK;
    H->poisoned = true;
    H->last_err.code = (int32_t)e.code;
    H->last_err.task = e.task;
    H->last_err.counter = e.counter;
    H->last_err.sm = e.sm;
    H->last_err.seen = e.seen;
    H->last_err.target = e.target;
    if (e.code == 3)
        return amk_set_error(AMK_ERR_POS_RANGE, "device token out of range (%u)", e.seen);
    return amk_set_error(AMK_ERR_TIMEOUT, "device wait timed out (code %u, task %d, counter "
                         "%d, sm %d, seen %u, needed %u)", e.code, e.task, e.counter, e.sm,
                         e.seen, e.target);
}

}  // namespace

extern "C" int amk_create(const amk_config *cfg, const amk_weights *w, const amk_options *opt,
                          void *cuda_stream, amk_handle **out)
{
    if (!cfg || !w || !out)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_create: NULL argument");
    *out = nullptr;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
        cudaGetLastError();
        return amk_set_error(AMK_ERR_NO_DEVICE, "amk_create: no CUDA device");
    }
    int rc = check_weights(cfg, w);
    if (rc != AMK_OK)
        return rc;
    amk_handle *H = new (std::nothrow) amk_handle();
    if (!H)
        return amk_set_error(AMK_ERR_OOM, "amk_create: out of host memory");
    cudaGetDevice(&H->device);
    H->stream = static_cast<cudaStream_t>(cuda_stream);
    H->guards_on = opt && opt->debug_checks > 0;
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, H->device);
    int n_sms = (opt && opt->n_sms > 0) ? opt->n_sms : sms;
    if (n_sms > sms) {
        delete H;
        return amk_set_error(AMK_ERR_INVALID_ARG, "n_sms %d > %d SMs on the device", n_sms, sms);
    }
    amk_validation_report rep;
    rc = amk_plan_create(cfg, opt, n_sms, &H->plan, &rep);
    if (rc != AMK_OK) {
        delete H;
        return rc;
    }
    const amk_plan *P = H->plan;
    const int q8 = P->cfg.quant == AMK_QUANT_W8A16 ? 1 : 0;
    const int qm = P->cfg.quant;  // 0 bf16, 1 int8, 2 int4
    cudaError_t e = amk_kernel_configure(P->smem_bytes, qm, P->att_e, P->generic, P->ffn_fused);
    if (e != cudaSuccess) {
        free_handle(H);
        return cuda_fail(e, "cudaFuncSetAttribute");
    }
    int per_sm = 0;
    e = amk_kernel_occupancy(P->smem_bytes, qm, P->att_e, P->generic, P->ffn_fused, &per_sm);
    if (e != cudaSuccess || per_sm < 1) {
        free_handle(H);
        return amk_set_error(AMK_ERR_LAUNCH, "kernel does not fit one SM (smem %d B)",
                             P->smem_bytes);
    }
    const amk_config &c = P->cfg;
    const int L = c.n_layers, nkv = c.n_kv_heads, hd = c.head_dim;
    const size_t part_floats = (size_t)nkv * P->opt.attn_splits * P->group * (hd + 2);
    const size_t qkv_f = (size_t)L * P->qkv_rows, part_f = (size_t)L * part_floats;
    const size_t attn_f = (size_t)L * c.n_heads * hd;
    const size_t h_f = (size_t)L * c.hidden, act_f = (size_t)L * c.ffn;
    H->kv_bytes = (size_t)L * 2 * nkv * c.max_ctx * hd * sizeof(uint16_t);
    // activations in one block: xacc (int64) | qkv | attn | xmid | xout
    // (flagged words, 8 bytes each) | act (32-bit flagged words) | part (fp32)
    const size_t xacc_b = P->ffn_fused ? (size_t)L * c.hidden * sizeof(long long) : 0;
    const size_t words = qkv_f + attn_f + 2 * h_f;
    H->fw_bytes = words * sizeof(uint64_t) + act_f * sizeof(uint32_t);
    H->act_bytes = xacc_b + H->fw_bytes + part_f * sizeof(float);
    float *act_block = nullptr;
    if ((rc = dalloc(H, &H->d_tasks, sizeof(TaskDesc) * P->tasks.size())) ||
        (rc = dalloc(H, &H->d_qoff, sizeof(int32_t) * P->queue_off.size())) ||
        (rc = dalloc(H, &H->d_ctr, sizeof(uint32_t) * (size_t)(P->n_counters + P->n_arrive))) ||
        (P->pos0 &&
         ((rc = dalloc(H, &H->d_tasks0, sizeof(TaskDesc) * P->pos0->tasks.size())) ||
          (rc = dalloc(H, &H->d_qoff0, sizeof(int32_t) * P->pos0->queue_off.size())) ||
          (rc = dalloc(H, &H->d_ctr0, sizeof(uint32_t) * (size_t)P->pos0->n_counters)))) ||
        (rc = dalloc(H, &H->d_err, sizeof(ErrorWord))) ||
        (rc = dalloc(H, &act_block, H->act_bytes)) ||
        (rc = dalloc(H, &H->d_logits, sizeof(float) * (size_t)c.vocab)) ||
        (rc = dalloc(H, &H->d_argkey, 2 * sizeof(unsigned long long))) ||
        (P->ffn_fused &&
         (rc = dalloc(H, &H->d_dpack, (size_t)L * c.hidden * c.ffn * (q8 ? 1 : 2)))) ||
        (rc = dalloc(H, &H->d_kv, H->kv_bytes)) ||
        (P->opt.profile &&
         (rc = dalloc(H, &H->d_prof, sizeof(unsigned long long) * (size_t)n_sms *
                                         amk::kProfKinds * amk::kProfFields)))) {
        free_handle(H);
        return rc;
    }
    H->d_act_block = act_block;
    H->d_xacc = P->ffn_fused ? reinterpret_cast<long long *>(act_block) : nullptr;
    H->d_qkv = reinterpret_cast<uint64_t *>(reinterpret_cast<char *>(act_block) + xacc_b);
    H->d_attn = H->d_qkv + qkv_f;
    H->d_xmid = H->d_attn + attn_f;
    H->d_xout = H->d_xmid + h_f;
    H->d_act = reinterpret_cast<uint32_t *>(H->d_xout + h_f);
    H->d_part = reinterpret_cast<float *>(H->d_act + act_f);
    if ((e = cudaMallocHost(&H->h_err, sizeof(ErrorWord))) != cudaSuccess ||
        (e = cudaMallocHost(&H->h_key, 2 * sizeof(unsigned long long))) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&H->err_ev, cudaEventDisableTiming)) != cudaSuccess) {
        free_handle(H);
        return cuda_fail(e, "host buffers");
    }
    // W4A16: pack every int4 matrix (codes and group scales of a row together)
    // into one allocation, and resolve the tasks against the packed copies
    amk_weights wq4 = *w;
    std::vector<const void *> q4_ptrs;
    if (qm == AMK_QUANT_W4A16) {
        const int hh = c.hidden, qr = c.n_heads * c.head_dim, kr = c.n_kv_heads * c.head_dim;
        const int F = c.ffn;
        const int rows7[7] = {qr, kr, kr, hh, F, F, hh};
        const int ks7[7] = {hh, hh, hh, qr, hh, hh, F};
        const void *const *mats[7] = {w->wq, w->wk, w->wv, w->wo, w->wgate, w->wup, w->wdown};
        const void *const *scs[7] = {w->sq, w->sk, w->sv, w->so, w->sgate, w->sup, w->sdown};
        size_t total = 0;
        for (int m = 0; m < 7; ++m)
            total += (size_t)L * rows7[m] * amk::q4_row_bytes(ks7[m]);
        if (!c.tied_embeddings)
            total += (size_t)c.vocab * amk::q4_row_bytes(hh);
        if ((rc = dalloc(H, &H->d_q4, total))) {
            free_handle(H);
            return rc;
        }
        q4_ptrs.resize((size_t)7 * L);
        uint8_t *dst = static_cast<uint8_t *>(H->d_q4);
        for (int m = 0; m < 7; ++m)
            for (int l = 0; l < L; ++l) {
                if ((e = amk_pack_q4(mats[m][l], scs[m][l], dst, rows7[m], ks7[m], H->stream)) !=
                    cudaSuccess) {
                    free_handle(H);
                    return cuda_fail(e, "pack int4 weights");
                }
                q4_ptrs[(size_t)m * L + l] = dst;
                dst += (size_t)rows7[m] * amk::q4_row_bytes(ks7[m]);
            }
        if (!c.tied_embeddings) {
            if ((e = amk_pack_q4(w->lm_head, w->lm_head_scale, dst, c.vocab, hh, H->stream)) !=
                cudaSuccess) {
                free_handle(H);
                return cuda_fail(e, "pack int4 LM head");
            }
            wq4.lm_head = dst;
        }
        const void *const *packed[7];
        for (int m = 0; m < 7; ++m)
            packed[m] = q4_ptrs.data() + (size_t)m * L;
        wq4.wq = packed[0], wq4.wk = packed[1], wq4.wv = packed[2], wq4.wo = packed[3];
        wq4.wgate = packed[4], wq4.wup = packed[5], wq4.wdown = packed[6];
    }
    const amk_weights *wr = qm == AMK_QUANT_W4A16 ? &wq4 : w;
    std::vector<TaskDesc> resolved(P->tasks.size());
    for (size_t t = 0; t < resolved.size(); ++t)
        amk_resolve_task(P, wr, H->d_kv, (int)t, &resolved[t], P->ffn_fused ? 1 : 0);
    // fused FFN: the handle's packed copy of every layer's Wdown
    for (int l = 0; P->ffn_fused && l < L; ++l) {
        const size_t lb = (size_t)c.hidden * c.ffn * (q8 ? 1 : 2);
        if ((e = amk_pack_down(w->wdown[l], static_cast<uint8_t *>(H->d_dpack) + l * lb,
                               c.hidden, c.ffn, q8 ? 1 : 2, H->stream)) != cudaSuccess) {
            free_handle(H);
            return cuda_fail(e, "pack Wdown");
        }
    }
    if (H->guards_on && (rc = check_task_records(P, resolved, H->d_kv, H->kv_bytes)) != AMK_OK) {
        free_handle(H);
        return rc;
    }
    if ((e = cudaMemcpyAsync(H->d_tasks, resolved.data(), sizeof(TaskDesc) * resolved.size(),
                             cudaMemcpyHostToDevice, H->stream)) != cudaSuccess ||
        (e = cudaMemcpyAsync(H->d_qoff, P->queue_off.data(),
                             sizeof(int32_t) * P->queue_off.size(), cudaMemcpyHostToDevice,
                             H->stream)) != cudaSuccess) {
        free_handle(H);
        return cuda_fail(e, "upload schedule");
    }
    std::vector<TaskDesc> resolved0(P->pos0 ? P->pos0->tasks.size() : 0);
    for (size_t t = 0; t < resolved0.size(); ++t)
        amk_resolve_task(P->pos0, wr, H->d_kv, (int)t, &resolved0[t], P->pos0->ffn_fused ? 1 : 0);
    if (H->guards_on && P->pos0 &&
        (rc = check_task_records(P->pos0, resolved0, H->d_kv, H->kv_bytes)) != AMK_OK) {
        free_handle(H);
        return rc;
    }
    if (P->pos0 &&
        ((e = cudaMemcpyAsync(H->d_tasks0, resolved0.data(), sizeof(TaskDesc) * resolved0.size(),
                              cudaMemcpyHostToDevice, H->stream)) != cudaSuccess ||
         (e = cudaMemcpyAsync(H->d_qoff0, P->pos0->queue_off.data(),
                              sizeof(int32_t) * P->pos0->queue_off.size(),
                              cudaMemcpyHostToDevice, H->stream)) != cudaSuccess)) {
        free_handle(H);
        return cuda_fail(e, "upload schedule");
    }
    if ((rc = zero_state(H)) != AMK_OK) {
        free_handle(H);
        return rc;
    }
    if ((e = cudaStreamSynchronize(H->stream)) != cudaSuccess) {  // also frees `resolved`'s use
        free_handle(H);
        return cuda_fail(e, "amk_create");
    }
    KParams &k = H->kp;
    k.tasks = H->d_tasks;
    k.queue_off = H->d_qoff;
    k.counters = H->d_ctr;
    k.err = H->d_err;
    k.embed = static_cast<const uint16_t *>(w->embed);
    k.qkv = H->d_qkv;
    k.part = H->d_part;
    k.attn = H->d_attn;
    k.arrive = H->d_ctr + P->n_counters;
    k.xmid = H->d_xmid;
    k.xout = H->d_xout;
    k.act = H->d_act;
    k.xacc = H->d_xacc;
    k.dmaps = nullptr;
    k.dpack = static_cast<const uint8_t *>(H->d_dpack);
    k.ffn_fused = P->ffn_fused;
    k.ffn_box_rows = P->ffn_box_rows;
    k.logits = H->d_logits;
    k.argkey = H->d_argkey;
    k.kv = H->d_kv;
    k.hidden = c.hidden;
    k.n_layers = L;
    k.n_heads = c.n_heads;
    k.n_kv_heads = nkv;
    k.head_dim = hd;
    k.ffn = c.ffn;
    k.vocab = c.vocab;
    k.max_ctx = c.max_ctx;
    k.qkv_rows = P->qkv_rows;
    k.group = P->group;
    k.attn_splits = P->opt.attn_splits;
    k.quant = qm;
    k.tied = c.tied_embeddings ? 1 : 0;
    k.rms_eps = c.rms_eps;
    k.rope_theta = c.rope_theta;
    k.ring_stages = P->opt.ring_stages;
    k.stage_bytes = P->opt.stage_bytes;
    k.vec_floats = P->vec_floats;
    k.att_lph = P->att_lph;
    k.att_hpb = P->att_hpb;
    k.att_e = P->att_e;
    k.att_pg = P->att_pg;
    k.generic = P->generic;
    k.timeout_ns = (uint64_t)P->opt.wait_timeout_us * 1000ull;
    k.skip_signal_task = P->opt.debug_skip_signal_task;
    k.flagged = P->flagged;
    k.lookahead = (uint32_t)std::max(0, P->opt.l2_prefetch_kb) * 1024u;
    k.inflight = amk_inflight_bytes(&P->opt);
    k.piece = amk_piece_bytes(&P->opt);
    k.prof = H->d_prof;
    *out = H;
    return AMK_OK;
}

extern "C" void amk_destroy(amk_handle *h) { free_handle(h); }

extern "C" int amk_reset_kv(amk_handle *h)
{
    if (!h)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_reset_kv: NULL handle");
    return zero_state(h);
}

namespace {

// Non-blocking look at the error word copied after an earlier step.
int poll_pending_error(amk_handle *H)
{
    if (!H->err_pending)
        return AMK_OK;
    if (cudaEventQuery(H->err_ev) != cudaSuccess) {
        cudaGetLastError();  // clear cudaErrorNotReady
        return AMK_OK;
    }
    H->err_pending = false;
    return absorb_error(H, *H->h_err);
}

int launch_step(amk_handle *H, int32_t token_id, int32_t pos, float *logits_dev,
                bool will_sync)
{
    if (!H)
        return amk_set_error(AMK_ERR_INVALID_ARG, "NULL handle");
    int rc = poll_pending_error(H);
    if (rc != AMK_OK)
        return rc;
    if (H->poisoned)
        return amk_set_error(AMK_ERR_POISONED, "handle poisoned; call amk_reset_kv");
    const amk_config &c = H->plan->cfg;
    if (pos < 0 || pos >= c.max_ctx)
        return amk_set_error(AMK_ERR_POS_RANGE, "pos %d outside [0, %d)", pos, c.max_ctx);
    if (token_id >= c.vocab || token_id < -1)
        return amk_set_error(AMK_ERR_POS_RANGE, "token %d outside [0, %d)", token_id, c.vocab);
    if (token_id == -1 && H->epoch == 0)
        return amk_set_error(AMK_ERR_INVALID_ARG, "token -1 needs a previous step");
    if (logits_dev && ((uintptr_t)logits_dev % 4))
        return amk_set_error(AMK_ERR_INVALID_ARG, "logits_dev misaligned");
    KParams k = H->kp;
    k.pos = pos;
    k.token = token_id;
    k.att_chunk = amk::attn_chunk_len(pos + 1, H->plan->opt.attn_splits);
    k.att_P = H->plan->opt.stage_bytes / (4 * c.head_dim);
    // counter epochs count the steps each schedule ran (parity counts all)
    k.epoch = H->epoch - H->epoch0;
    const bool at0 = pos == 0 && H->plan->pos0;
    if (at0) {  // the position-0 schedule, with its own counters
        k.tasks = H->d_tasks0;
        k.queue_off = H->d_qoff0;
        k.counters = H->d_ctr0;
        k.epoch = H->epoch0;
    }
    k.arrive_base = H->arrive_base;
    k.parity = (int32_t)(H->epoch & 1u);
    // a fresh tag per step; when the 32-bit tag runs out, every flagged word
    // is cleared (stream-ordered before this launch) and the tags start over
    if (H->tag == 0xFFFFFFFFu) {
        cudaError_t ce = cudaMemsetAsync(H->d_qkv, 0, H->fw_bytes, H->stream);
        if (ce != cudaSuccess)
            return cuda_fail(ce, "flagged words clear");
        H->tag = 0;
    }
    k.tag = H->tag + 1;
    if (logits_dev)
        k.logits = logits_dev;
    if (H->d_prof) {
        cudaError_t pe = cudaMemsetAsync(H->d_prof, 0,
                                         sizeof(unsigned long long) * (size_t)H->plan->n_sms *
                                             amk::kProfKinds * amk::kProfFields,
                                         H->stream);
        if (pe != cudaSuccess)
            return cuda_fail(pe, "profile clear");
    }
    cudaError_t e = amk::amk_kernel_launch(&k, H->plan->n_sms, H->plan->smem_bytes, H->stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return amk_set_error(e == cudaErrorCooperativeLaunchTooLarge ? AMK_ERR_LAUNCH
                                                                      : AMK_ERR_CUDA,
                             "cooperative launch: %s", cudaGetErrorString(e));
    }
    H->epoch += 1;
    H->tag += 1;
    if (at0)
        H->epoch0 += 1;
    {  // non-empty attention chunks of this step: each arrives once unless alone
        const int C = H->plan->opt.attn_splits, n = pos + 1;
        const int chunk = amk::attn_chunk_len(n, C), nne = (n + chunk - 1) / chunk;
        if (nne > 1)
            H->arrive_base += (uint32_t)nne;
    }
    // The error word is read back when the caller synchronises, and every 32
    // asynchronous steps otherwise (a failed step makes later kernels exit at
    // once, so a late look costs no device time).
    if (will_sync || (H->epoch % 32u) == 0u) {
        e = cudaMemcpyAsync(H->h_err, H->d_err, sizeof(ErrorWord), cudaMemcpyDeviceToHost,
                            H->stream);
        if (e == cudaSuccess && !will_sync)
            e = cudaEventRecord(H->err_ev, H->stream);
        if (e != cudaSuccess)
            return cuda_fail(e, "error word copy");
        H->err_pending = !will_sync;
    }
    return AMK_OK;
}

int finish_sync(amk_handle *H, int32_t *argmax_host)
{
    const int parity = (int)((H->epoch - 1) & 1u);
    cudaError_t e = cudaSuccess;
    if (argmax_host)
        e = cudaMemcpyAsync(H->h_key, H->d_argkey + parity, sizeof(unsigned long long),
                            cudaMemcpyDeviceToHost, H->stream);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(H->stream);
    if (e != cudaSuccess)
        return cuda_fail(e, "decode step");
    H->err_pending = false;
    int rc = absorb_error(H, *H->h_err);
    if (rc != AMK_OK)
        return rc;
    if (argmax_host)
        *argmax_host = (int32_t)(0xFFFFFFFFu - (uint32_t)(*H->h_key & 0xFFFFFFFFull));
    return AMK_OK;
}

}  // namespace

extern "C" int amk_decode_step(amk_handle *h, int32_t token_id, int32_t pos, float *logits_dev,
                               int32_t *argmax_host)
{
    int rc = launch_step(h, token_id, pos, logits_dev, argmax_host != nullptr);
    if (rc != AMK_OK || !argmax_host)
        return rc;
    return finish_sync(h, argmax_host);
}

extern "C" int amk_decode_step_host(amk_handle *h, int32_t token_id, int32_t pos,
                                    float *logits_host, int32_t *argmax_host)
{
    int rc = launch_step(h, token_id, pos, nullptr, true);
    if (rc != AMK_OK)
        return rc;
    if (logits_host) {
        cudaError_t e = cudaMemcpyAsync(logits_host, h->d_logits,
                                        sizeof(float) * (size_t)h->plan->cfg.vocab,
                                        cudaMemcpyDeviceToHost, h->stream);
        if (e != cudaSuccess)
            return cuda_fail(e, "logits copy");
    }
    return finish_sync(h, argmax_host);
}

extern "C" int amk_get_kv(amk_handle *h, int32_t layer, void **k_dev, void **v_dev)
{
    if (!h || layer < 0 || layer >= h->plan->cfg.n_layers)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_get_kv: bad handle or layer");
    const amk_config &c = h->plan->cfg;
    const size_t blk = (size_t)c.n_kv_heads * c.max_ctx * c.head_dim;
    if (k_dev)
        *k_dev = h->d_kv + ((size_t)layer * 2 + 0) * blk;
    if (v_dev)
        *v_dev = h->d_kv + ((size_t)layer * 2 + 1) * blk;
    return AMK_OK;
}

extern "C" int amk_get_logits(amk_handle *h, float **logits_dev)
{
    if (!h || !logits_dev)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_get_logits: NULL argument");
    *logits_dev = h->d_logits;
    return AMK_OK;
}

extern "C" int amk_plan_get_stats(const amk_plan *P, amk_plan_stats *o)
{
    if (!P || !o)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_plan_get_stats: NULL argument");
    memset(o, 0, sizeof *o);
    o->n_tasks = (int32_t)P->tasks.size();
    o->n_counters = P->n_counters;
    o->n_sms = P->n_sms;
    o->ring_stages = P->opt.ring_stages;
    o->stage_bytes = P->opt.stage_bytes;
    o->attn_splits = P->opt.attn_splits;
    o->smem_bytes = P->smem_bytes;
    o->threads_per_cta = amk::kThreads;
    o->weight_bytes = P->weight_bytes;
    o->kv_row_bytes = P->kv_row_bytes;
    o->flagged_waits = P->flagged;
    o->ffn_fused = P->ffn_fused;
    return AMK_OK;
}

extern "C" int amk_get_stats(amk_handle *h, amk_plan_stats *o)
{
    if (!h || !o)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_get_stats: NULL argument");
    const int rc = amk_plan_get_stats(h->plan, o);
    if (rc == AMK_OK)
        o->epoch = h->epoch;
    return rc;
}

extern "C" int amk_get_workspace(amk_handle *h, amk_workspace *out)
{
    if (!h || !out)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_get_workspace: NULL argument");
    out->qkv = h->d_qkv;
    out->xmid = h->d_xmid;
    out->xout = h->d_xout;
    out->act = h->d_act;
    out->qkv_rows = h->plan->qkv_rows;
    return AMK_OK;
}

extern "C" int amk_get_profile(amk_handle *h, uint64_t *out, int64_t n_u64)
{
    if (!h || !out || !h->d_prof)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_get_profile: profiling is off or NULL");
    const int64_t need = (int64_t)h->plan->n_sms * amk::kProfKinds * amk::kProfFields;
    if (n_u64 < need)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_get_profile: need %lld entries",
                             (long long)need);
    cudaError_t e = cudaMemcpyAsync(out, h->d_prof, sizeof(uint64_t) * (size_t)need,
                                    cudaMemcpyDeviceToHost, h->stream);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(h->stream);
    if (e != cudaSuccess)
        return cuda_fail(e, "amk_get_profile");
    return AMK_OK;
}

extern "C" int amk_check_guards(amk_handle *h, int32_t *n_bad)
{
    if (!h || !n_bad)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_check_guards: NULL argument");
    if (!h->guards_on)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_check_guards: the handle was created "
                             "without debug_checks");
    cudaError_t e = cudaStreamSynchronize(h->stream);
    int32_t bad = 0;
    std::vector<uint8_t> buf(kGuardBytes);
    for (const void *g : h->guards) {
        if (e == cudaSuccess)
            e = cudaMemcpy(buf.data(), g, kGuardBytes, cudaMemcpyDeviceToHost);
        if (e != cudaSuccess)
            break;
        for (uint8_t v : buf)
            if (v != (uint8_t)kGuardByte) {
                ++bad;
                break;
            }
    }
    if (e != cudaSuccess)
        return cuda_fail(e, "amk_check_guards");
    *n_bad = bad;
    return AMK_OK;
}

extern "C" int amk_get_error_info(amk_handle *h, amk_error_info *out)
{
    if (!h || !out)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_get_error_info: NULL argument");
    *out = h->last_err;
    return AMK_OK;
}
