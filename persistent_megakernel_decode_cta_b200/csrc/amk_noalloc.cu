// amk_noalloc.cu -- a decode step that allocates no memory.
//
// Some callers cannot call cudaMalloc: plugins inside an inference server or
// a framework whose allocator owns every device byte (a stray cudaMalloc
// breaks its accounting and can fail when the pool has reserved the rest of
// the GPU), and latency-critical loops where cudaMalloc/cudaFree would stall
// on an implicit device synchronisation.  amk_create allocates the KV cache
// and the workspace, so those callers use amk_decode_step_noalloc instead:
// the caller owns the weights, the KV cache and the logits, and the step's
// scratch (task table, counters, error word, argmax key, activations) lives
// in the fixed array g_scratch below, which exists once per GPU from the
// moment the library's device code is loaded until the process exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "amk.h"
#include "amk_internal.h"
#include "amk_plan.h"

extern "C" int amk_kernel_smem_bytes(int ring_stages, int stage_bytes, int vec_floats);
extern "C" cudaError_t amk_kernel_configure(int smem_bytes, int quant, int att_e, int generic,
                                            int fused);
namespace amk {
extern "C" cudaError_t amk_kernel_launch(const KParams *p, int n_ctas, int smem_bytes,
                                         cudaStream_t stream);
}

namespace {

constexpr size_t kScratchBytes = AMK_NOALLOC_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

struct Layout {
    size_t tasks, qoff, ctr, err, argkey, qkv, part, attn, xmid, xout, act, xacc, dmaps, total;
};

Layout layout_of(const amk_plan &P)
{
    const amk_config &c = P.cfg;
    const size_t L = (size_t)c.n_layers;
    const size_t part = (size_t)c.n_kv_heads * P.opt.attn_splits * P.group * (c.head_dim + 2);
    Layout o{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t at = off;
        off = up256(off + bytes);
        return at;
    };
    o.tasks = take(sizeof(amk::TaskDesc) * P.tasks.size());
    o.qoff = take(sizeof(int32_t) * P.queue_off.size());
    o.ctr = take(sizeof(uint32_t) * (size_t)(P.n_counters + P.n_arrive));
    o.err = take(sizeof(amk::ErrorWord));
    o.argkey = take(2 * sizeof(unsigned long long));
    // flagged words (8 bytes each) from qkv to the end of act
    o.qkv = take(sizeof(uint64_t) * L * P.qkv_rows);
    o.attn = take(sizeof(uint64_t) * L * c.n_heads * c.head_dim);
    o.xmid = take(sizeof(uint64_t) * L * c.hidden);
    o.xout = take(sizeof(uint64_t) * L * c.hidden);
    o.act = take(sizeof(uint32_t) * L * c.ffn);
    o.part = take(sizeof(float) * L * part);
    o.xacc = take(P.ffn_fused ? sizeof(long long) * L * c.hidden : 0);
    o.dmaps = take(P.ffn_fused ? 128 * L : 0);
    o.total = off;
    return o;
}

// Device address of g_scratch on the current device.  In host code the name
// g_scratch is only a host-side stand-in, so the kernel gets the address the
// runtime reports.  The first call on a device is the set-up (it loads the
// library's device code there if that has not happened yet); every call looks
// the address up again, a host-side query, so that it stays right after the
// device's context has been reset (which reloads the device code, possibly
// at another address).
int scratch_address(unsigned char **out)
{
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p)
        return amk_set_error(AMK_ERR_CUDA, "cudaGetSymbolAddress(g_scratch): %s",
                             cudaGetErrorString(e));
    *out = static_cast<unsigned char *>(p);
    return AMK_OK;
}

// What the static array holds from the last call on a device: the plan and
// the pointers its task table was resolved against, and the CUDA context it
// was written in (a context id is never reused in a process, so a reset of
// the device shows as a new id).  A call with the same key finds the task
// table, queue offsets and tensor maps in place and uploads nothing but the
// cleared counters; any other call rewrites them.
struct UploadKey {
    uint64_t plan_uid = 0, ctx_id = 0, wsig = 0;
    const void *kv = nullptr;
    unsigned char *base = nullptr;
};
constexpr int kMaxDevices = 64;
std::mutex g_upload_mu;
UploadKey g_uploaded[kMaxDevices];
// The tag of the last step each device's array ran (every call takes the
// next one), and the plan that ran it.  Plans lay the array out differently:
// where this plan keeps flagged words another may have kept anything (a
// fixed-point residual's high half is a small integer, like a tag), so the
// flagged words are cleared whenever the plan changes.
uint32_t g_fw_tag[kMaxDevices];
uint64_t g_fw_plan[kMaxDevices];

// FNV-1a over the weight pointers the task table holds.
uint64_t weights_signature(const amk_config &c, const amk_weights *w)
{
    uint64_t h = 1469598103934665603ull;
    auto mix = [&](const void *p) {
        uint64_t v = (uint64_t)(uintptr_t)p;
        for (int i = 0; i < 8; ++i, v >>= 8) {
            h ^= (v & 0xff);
            h *= 1099511628211ull;
        }
    };
    mix(w->embed), mix(w->final_norm), mix(w->lm_head), mix(w->lm_head_scale);
    const void *const *arr[16] = {w->attn_norm, w->ffn_norm, w->wq,    w->wk,
                                  w->wv,        w->wo,       w->wgate, w->wup,
                                  w->wdown,     w->sq,       w->sk,    w->sv,
                                  w->so,        w->sgate,    w->sup,   w->sdown};
    for (int a = 0; a < 16; ++a)
        for (int l = 0; l < c.n_layers; ++l)
            mix(arr[a] ? arr[a][l] : nullptr);
    return h;
}

// The id of the calling thread's current CUDA context (0 if unknown: then
// every call uploads).
uint64_t current_context_id()
{
    typedef CUresult (*GetCurrent)(CUcontext *);
    typedef CUresult (*GetId)(CUcontext, unsigned long long *);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static bool looked = false;
    if (!looked) {
        void *f1 = nullptr, *f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) ==
                cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
            q2 == cudaDriverEntryPointSuccess) {
            get_current = reinterpret_cast<GetCurrent>(f1);
            get_id = reinterpret_cast<GetId>(f2);
        }
        looked = true;
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

bool ok16(const void *p) { return p && ((uintptr_t)p % 16) == 0; }

int fail_cuda(cudaError_t e, const char *what)
{
    return amk_set_error(AMK_ERR_CUDA, "amk_decode_step_noalloc: %s: %s", what,
                         cudaGetErrorString(e));
}

}  // namespace

extern "C" int amk_decode_step_noalloc(const amk_plan *plan, const amk_weights *w,
                                       void *kv_cache, int32_t token_id, int32_t pos,
                                       float *logits_dev, int32_t *argmax_host,
                                       void *cuda_stream)
{
    if (!plan || !w || !ok16(kv_cache) || !logits_dev || ((uintptr_t)logits_dev % 4))
        return amk_set_error(AMK_ERR_INVALID_ARG,
                             "amk_decode_step_noalloc: NULL or misaligned argument");
    const amk_plan &P = *plan;
    const amk_config &c = P.cfg;
    if (pos < 0 || pos >= c.max_ctx || token_id < 0 || token_id >= c.vocab)
        return amk_set_error(AMK_ERR_POS_RANGE, "amk_decode_step_noalloc: token %d / pos %d "
                             "out of range", token_id, pos);
    const bool q8 = c.quant == AMK_QUANT_W8A16;
    if (c.quant == AMK_QUANT_W4A16)
        return amk_set_error(AMK_ERR_UNSUPPORTED, "amk_decode_step_noalloc: int4 weights are "
                             "packed by amk_create, which allocates; use amk_create");
    if (!ok16(w->embed) || !ok16(w->final_norm) || !w->attn_norm || !w->ffn_norm ||
        (!c.tied_embeddings && (!ok16(w->lm_head) || (q8 && !w->lm_head_scale))))
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_decode_step_noalloc: weights");
    const void *const *mats[7] = {w->wq, w->wk, w->wv, w->wo, w->wgate, w->wup, w->wdown};
    const void *const *scs[7] = {w->sq, w->sk, w->sv, w->so, w->sgate, w->sup, w->sdown};
    for (int m = 0; m < 7; ++m)
        if (!mats[m] || (q8 && !scs[m]))
            return amk_set_error(AMK_ERR_INVALID_ARG, "amk_decode_step_noalloc: weights");
    const Layout lay = layout_of(P);
    if (lay.total > kScratchBytes)
        return amk_set_error(AMK_ERR_UNSUPPORTED,
                             "amk_decode_step_noalloc: this model needs %zu bytes of scratch, "
                             "more than the %zu-byte static array; use amk_create",
                             lay.total, kScratchBytes);
    if (P.is_pos0 && pos != 0)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_decode_step_noalloc: the position-0 "
                             "schedule runs only steps at position 0 (pos %d)", pos);
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    {
        // the schedule uploads below read host stack buffers; a captured
        // graph would keep pointers to them
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        const cudaError_t ce = cudaStreamIsCapturing(st, &cs);
        if (ce != cudaSuccess)
            return fail_cuda(ce, "cudaStreamIsCapturing");
        if (cs != cudaStreamCaptureStatusNone)
            return amk_set_error(AMK_ERR_UNSUPPORTED, "amk_decode_step_noalloc: the stream is "
                                 "capturing; the call uploads its schedule from host stack "
                                 "memory and does nothing under capture");
    }
    int dev = 0, sms = 0;
    cudaError_t de = cudaGetDevice(&dev);
    if (de == cudaSuccess)
        de = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (de != cudaSuccess)
        return amk_set_error(AMK_ERR_NO_DEVICE, "amk_decode_step_noalloc: %s",
                             cudaGetErrorString(de));
    if (P.n_sms > sms)
        return amk_set_error(AMK_ERR_INVALID_ARG, "plan made for %d SMs, device has %d",
                             P.n_sms, sms);
    unsigned char *base = nullptr;
    int rc = scratch_address(&base);
    if (rc != AMK_OK)
        return rc;
    cudaError_t e;
    // per-layer pointers must all be present before any task is resolved
    for (int l = 0; l < c.n_layers; ++l) {
        if (!ok16(w->attn_norm[l]) || !ok16(w->ffn_norm[l]))
            return amk_set_error(AMK_ERR_INVALID_ARG, "layer %d norm NULL or misaligned", l);
        for (int m = 0; m < 7; ++m)
            if (!ok16(mats[m][l]) || (q8 && !scs[m][l]))
                return amk_set_error(AMK_ERR_INVALID_ARG, "layer %d weight %d", l, m);
    }
    // schedule tables with resolved pointers (skipped when the array already
    // holds this plan's, resolved against these pointers in this context)
    const UploadKey ukey{P.uid, current_context_id(), weights_signature(c, w), kv_cache, base};
    bool cached = false;
    if (dev >= 0 && dev < kMaxDevices && ukey.ctx_id != 0) {
        std::lock_guard<std::mutex> lock(g_upload_mu);
        const UploadKey &u = g_uploaded[dev];
        cached = u.plan_uid == ukey.plan_uid && u.ctx_id == ukey.ctx_id && u.wsig == ukey.wsig &&
                 u.kv == ukey.kv && u.base == ukey.base;
        g_uploaded[dev] = UploadKey{};  // rewritten below; valid again once it is
    }
    if (!cached) {
        // in batches through a stack buffer (pageable sources: cudaMemcpyAsync
        // stages them before returning, so the buffer can be reused at once)
        e = cudaMemcpyAsync(base + lay.qoff, P.queue_off.data(), sizeof(int32_t) * P.queue_off.size(),
                            cudaMemcpyHostToDevice, st);
        if (e != cudaSuccess)
            return fail_cuda(e, "schedule upload");
        amk::TaskDesc batch[64];
        const uint16_t *kv = static_cast<const uint16_t *>(kv_cache);
        const int T = (int)P.tasks.size();
        for (int t0 = 0; t0 < T; t0 += 64) {
            const int n = T - t0 < 64 ? T - t0 : 64;
            for (int i = 0; i < n; ++i)
                amk_resolve_task(&P, w, kv, t0 + i, &batch[i], 0);
            e = cudaMemcpyAsync(base + lay.tasks + sizeof(amk::TaskDesc) * (size_t)t0, batch,
                                sizeof(amk::TaskDesc) * (size_t)n, cudaMemcpyHostToDevice, st);
            if (e != cudaSuccess)
                return fail_cuda(e, "schedule upload");
        }
        // tensor maps of Wdown (fused FFN), through a stack buffer
        if (P.ffn_fused) {
            alignas(64) unsigned char mbuf[128 * 16];
            for (int l0 = 0; l0 < c.n_layers; l0 += 16) {
                const int n = c.n_layers - l0 < 16 ? c.n_layers - l0 : 16;
                const int mrc = amk_encode_down_maps(&P, w, l0, n, mbuf);
                if (mrc != AMK_OK)
                    return mrc;
                e = cudaMemcpyAsync(base + lay.dmaps + 128 * (size_t)l0, mbuf, 128 * (size_t)n,
                                    cudaMemcpyHostToDevice, st);
                if (e != cudaSuccess)
                    return fail_cuda(e, "tensor map upload");
            }
        }
    }
    if (dev >= 0 && dev < kMaxDevices && ukey.ctx_id != 0) {
        std::lock_guard<std::mutex> lock(g_upload_mu);
        g_uploaded[dev] = ukey;
    }
    // what must start at zero: counters, error word, argmax keys
    e = cudaMemsetAsync(base + lay.ctr, 0, lay.qkv - lay.ctr, st);
    if (e != cudaSuccess)
        return fail_cuda(e, "scratch clear");
    // this step's tag; when the device's tags run out, the plan changed, or
    // the device ordinal is beyond the table, the flagged words are cleared
    // first
    uint32_t tag = 1;
    bool clear = true;
    if (dev >= 0 && dev < kMaxDevices) {
        std::lock_guard<std::mutex> lock(g_upload_mu);
        tag = ++g_fw_tag[dev];
        clear = tag == 0 || g_fw_plan[dev] != P.uid;
        g_fw_plan[dev] = P.uid;
        if (tag == 0)
            tag = g_fw_tag[dev] = 1;
    }
    if (clear) {
        e = cudaMemsetAsync(base + lay.qkv, 0, lay.part - lay.qkv, st);
        if (e != cudaSuccess)
            return fail_cuda(e, "scratch clear");
    }

    amk::KParams k{};
    k.tasks = reinterpret_cast<const amk::TaskDesc *>(base + lay.tasks);
    k.queue_off = reinterpret_cast<const int32_t *>(base + lay.qoff);
    k.counters = reinterpret_cast<uint32_t *>(base + lay.ctr);
    k.err = reinterpret_cast<amk::ErrorWord *>(base + lay.err);
    k.embed = static_cast<const uint16_t *>(w->embed);
    k.qkv = reinterpret_cast<uint64_t *>(base + lay.qkv);
    k.part = reinterpret_cast<float *>(base + lay.part);
    k.attn = reinterpret_cast<uint64_t *>(base + lay.attn);
    k.arrive = reinterpret_cast<uint32_t *>(base + lay.ctr) + P.n_counters;
    k.xmid = reinterpret_cast<uint64_t *>(base + lay.xmid);
    k.xout = reinterpret_cast<uint64_t *>(base + lay.xout);
    k.act = reinterpret_cast<uint32_t *>(base + lay.act);
    k.xacc = reinterpret_cast<long long *>(base + lay.xacc);
    k.dmaps = base + lay.dmaps;
    k.dpack = nullptr;  // no room for a packed copy: the tensor maps read the caller's Wdown
    k.ffn_fused = P.ffn_fused;
    k.ffn_box_rows = P.ffn_box_rows;
    k.logits = logits_dev;
    k.argkey = reinterpret_cast<unsigned long long *>(base + lay.argkey);
    k.kv = static_cast<uint16_t *>(kv_cache);
    k.hidden = c.hidden;
    k.n_layers = c.n_layers;
    k.n_heads = c.n_heads;
    k.n_kv_heads = c.n_kv_heads;
    k.head_dim = c.head_dim;
    k.ffn = c.ffn;
    k.vocab = c.vocab;
    k.max_ctx = c.max_ctx;
    k.qkv_rows = P.qkv_rows;
    k.group = P.group;
    k.attn_splits = P.opt.attn_splits;
    k.quant = q8 ? 1 : 0;
    k.tied = c.tied_embeddings ? 1 : 0;
    k.rms_eps = c.rms_eps;
    k.rope_theta = c.rope_theta;
    k.ring_stages = P.opt.ring_stages;
    k.stage_bytes = P.opt.stage_bytes;
    k.vec_floats = P.vec_floats;
    k.att_lph = P.att_lph;
    k.att_hpb = P.att_hpb;
    k.att_e = P.att_e;
    k.att_pg = P.att_pg;
    k.generic = P.generic;
    k.pos = pos;
    k.token = token_id;
    k.att_chunk = amk::attn_chunk_len(pos + 1, P.opt.attn_splits);
    k.att_P = P.opt.stage_bytes / (4 * c.head_dim);
    k.epoch = 0;   // counters were cleared above
    k.arrive_base = 0;
    k.parity = 0;
    k.timeout_ns = (uint64_t)P.opt.wait_timeout_us * 1000ull;
    k.skip_signal_task = P.opt.debug_skip_signal_task;
    k.tag = tag;
    k.flagged = P.flagged;
    k.lookahead = (uint32_t)(P.opt.l2_prefetch_kb > 0 ? P.opt.l2_prefetch_kb : 0) * 1024u;
    k.inflight = amk_inflight_bytes(&P.opt);
    k.piece = amk_piece_bytes(&P.opt);
    e = amk_kernel_configure(P.smem_bytes, q8 ? 1 : 0, P.att_e, P.generic, P.ffn_fused);
    if (e != cudaSuccess)
        return fail_cuda(e, "cudaFuncSetAttribute");
    e = amk::amk_kernel_launch(&k, P.n_sms, P.smem_bytes, st);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return amk_set_error(e == cudaErrorCooperativeLaunchTooLarge ? AMK_ERR_LAUNCH
                                                                      : AMK_ERR_CUDA,
                             "amk_decode_step_noalloc: launch: %s", cudaGetErrorString(e));
    }
    if (!argmax_host)
        return AMK_OK;
    // pageable destinations: these copies complete before the calls return
    unsigned long long key = 0;
    amk::ErrorWord ew;
    e = cudaMemcpyAsync(&ew, base + lay.err, sizeof ew, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(&key, base + lay.argkey, sizeof key, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(st);
    if (e != cudaSuccess)
        return fail_cuda(e, "result copy");
    if (ew.code != 0)
        return amk_set_error(ew.code == 3 ? AMK_ERR_POS_RANGE : AMK_ERR_TIMEOUT,
                             "amk_decode_step_noalloc: device error %u (task %d, counter %d)",
                             ew.code, ew.task, ew.counter);
    *argmax_host = (int32_t)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
    return AMK_OK;
}
