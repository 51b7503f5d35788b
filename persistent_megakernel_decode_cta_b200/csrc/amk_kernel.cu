// amk_kernel.cu -- the persistent decode megakernel for sm_100a.
//
// One launch = one forward pass = one token ("RightNow-AI/AutoMegaKernel"
// README, opening summary).  One CTA per SM walks its own queue of tasks in a
// global topological order: wait on a counter -> run the task -> signal a
// counter (gist.science technical summary, "Methodologie", layer 0; paperfeed
// review, "How it works").  Producers only increment counters and consumers
// only wait for statically known thresholds (README, "Deadlock-free by
// construction").  Weights of upcoming tasks are prefetched while the current
// one computes (README, "Why a megakernel").
//
// B200 design (not the pages' sm_80..sm_120 design):
//  * 288 threads per CTA: 8 consumer warps compute, 1 producer warp streams.
//  * The producer walks the same queue AHEAD of the consumers and copies each
//    task's weight rows (or KV-cache rows) into a ring of shared-memory
//    stages with cp.async.bulk (TMA bulk copies) that complete on per-stage
//    mbarriers.  Weights never depend on activations, so the copies run
//    ahead across counter waits: the wait latency is hidden behind the ring.
//  * Consumers wait on the counter (ld.acquire.gpu spin with a time limit),
//    build the task's input vector in shared memory (RMSNorm / split-K
//    combine prologues, all from L2 with .cg loads), run the GEMV from the
//    ring with each warp owning a fixed K-slice whose activations sit in
//    registers, reduce with warp shuffles, apply the fused epilogue
//    (RoPE+KV append, SwiGLU, residual add, argmax), then release their
//    stores with red.release.gpu on the task's counter.
//  * Every wait is bounded (globaltimer + iteration cap); on expiry the CTA
//    records the failure, drains its own TMA copies and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "amk_internal.h"

namespace amk {
namespace {

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void bulk_g2s_nohint(void *dst, const void *src, uint32_t bytes,
                                                uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ uint64_t evict_first_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_release_add(uint32_t *p, uint32_t v)
{
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint64_t gtimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void consumer_bar()
{
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory");
}

// ------------------------------------------------------------- number formats
__device__ __forceinline__ float bf16_to_f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }
__device__ __forceinline__ uint16_t f_to_bf16(float f)
{
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
__device__ __forceinline__ float fp16_to_f(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// int8 -> float exactly: 0x4B000000 | (q + 128) is the float 2^23 + q + 128.
__device__ __forceinline__ float i8f(uint32_t biased_word, uint32_t sel)
{
    return __uint_as_float(__byte_perm(biased_word, 0x4B000000u, sel)) - 8388736.0f;
}

template <int ESZ>
__device__ __forceinline__ float fma_word(uint32_t w, const float *x, float acc)
{
    if constexpr (ESZ == 2) {
        acc = fmaf(__uint_as_float(w << 16), x[0], acc);
        acc = fmaf(__uint_as_float(w & 0xffff0000u), x[1], acc);
    } else {
        const uint32_t b = w ^ 0x80808080u;
        acc = fmaf(i8f(b, 0x7440), x[0], acc);
        acc = fmaf(i8f(b, 0x7441), x[1], acc);
        acc = fmaf(i8f(b, 0x7442), x[2], acc);
        acc = fmaf(i8f(b, 0x7443), x[3], acc);
    }
    return acc;
}

template <int ESZ, int VB>
__device__ __forceinline__ float vdot(const uint8_t *p, const float *x, float acc)
{
    constexpr int EW = 4 / ESZ;  // elements per 32-bit word
    if constexpr (VB == 16) {
        const uint4 w = *reinterpret_cast<const uint4 *>(p);
        acc = fma_word<ESZ>(w.x, x, acc);
        acc = fma_word<ESZ>(w.y, x + EW, acc);
        acc = fma_word<ESZ>(w.z, x + 2 * EW, acc);
        acc = fma_word<ESZ>(w.w, x + 3 * EW, acc);
    } else if constexpr (VB == 8) {
        const uint2 w = *reinterpret_cast<const uint2 *>(p);
        acc = fma_word<ESZ>(w.x, x, acc);
        acc = fma_word<ESZ>(w.y, x + EW, acc);
    } else {
        acc = fma_word<ESZ>(*reinterpret_cast<const uint32_t *>(p), x, acc);
    }
    return acc;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ------------------------------------------------------------ shared memory
struct SmemLayout {
    uint8_t *ring;        // ring_stages * stage_bytes
    float *vec;           // vec_floats: the task's input vector / scratch
    float *red;           // [kConsumerWarps][kMaxTaskRows]
    uint64_t *full;       // [kMaxStages]
    uint64_t *empty;      // [kMaxStages]
    int *flags;           // [0] abort, [1] token, [2..] scratch
    float *scr;           // 64 floats of reduction scratch
};

__device__ __forceinline__ SmemLayout smem_layout(uint8_t *base, const KParams &p)
{
    SmemLayout s;
    size_t off = 0;
    s.ring = base;
    off += (size_t)p.ring_stages * p.stage_bytes;
    s.vec = reinterpret_cast<float *>(base + off);
    off += (size_t)p.vec_floats * 4;
    s.red = reinterpret_cast<float *>(base + off);
    off += (size_t)kConsumerWarps * kMaxTaskRows * 4;
    s.full = reinterpret_cast<uint64_t *>(base + off);
    off += kMaxStages * 8;
    s.empty = reinterpret_cast<uint64_t *>(base + off);
    off += kMaxStages * 8;
    s.flags = reinterpret_cast<int *>(base + off);
    off += 16 * 4;
    s.scr = reinterpret_cast<float *>(base + off);
    return s;
}

// ------------------------------------------------------------- task geometry
// Both the producer and the consumers derive a task's chunk stream from its
// descriptor with this function, so they agree on every chunk.
struct Geom {
    int nchunks;
    // GEMV tiles
    const uint8_t *base0, *base1;  // row r0 of part 0 / part 1
    const uint16_t *scale0, *scale1;
    int K, esz, RB, rpc, R, nck;
    // attention tiles
    int j0, j1, pa, pb, P;
    const uint8_t *kb, *vb;
};

__device__ __forceinline__ int gcd16(int v)
{
    int g = 16;
    while (v % g)
        g >>= 1;
    return g;
}

__device__ Geom task_geom(const KParams &p, const TaskDesc &d)
{
    Geom g{};
    const int l = d.layer;
    const int q8 = p.quant;
    if (d.kind == TK_ATTN) {
        const int gi = d.r0, c = d.r1, hd = p.head_dim;
        const int n = p.pos + 1;
        const int chunk = (n + p.attn_splits - 1) / p.attn_splits;
        g.j0 = c * chunk;
        g.j1 = min(g.j0 + chunk, n);
        if (g.j1 < g.j0)
            g.j1 = g.j0;
        g.pa = g.j0;
        g.pb = max(g.pa, min(g.j1, p.pos));
        g.P = p.stage_bytes / (4 * hd);
        const size_t blk = (size_t)p.max_ctx * hd;
        const uint16_t *kbase = p.kv + (((size_t)l * 2 + 0) * p.n_kv_heads + gi) * blk;
        const uint16_t *vbase = p.kv + (((size_t)l * 2 + 1) * p.n_kv_heads + gi) * blk;
        g.kb = reinterpret_cast<const uint8_t *>(kbase);
        g.vb = reinterpret_cast<const uint8_t *>(vbase);
        g.nchunks = (g.pb - g.pa + g.P - 1) / g.P;
        return g;
    }
    const LayerPtrs *L = (d.kind == TK_LMHEAD) ? nullptr : &p.layers[l];
    const void *w0 = nullptr, *w1 = nullptr;
    const uint16_t *s0 = nullptr, *s1 = nullptr;
    int K = p.hidden, esz = q8 ? 1 : 2, parts = 1;
    switch (d.kind) {
    case TK_QKV:
        w0 = L->w[d.mat];
        s0 = L->s[d.mat];
        break;
    case TK_OPROJ:
        w0 = L->w[W_O];
        s0 = L->s[W_O];
        K = p.n_heads * p.head_dim;
        break;
    case TK_GATEUP:
        w0 = L->w[W_GATE];
        s0 = L->s[W_GATE];
        w1 = L->w[W_UP];
        s1 = L->s[W_UP];
        parts = 2;
        break;
    case TK_DOWN:
        w0 = L->w[W_DOWN];
        s0 = L->s[W_DOWN];
        K = p.ffn;
        break;
    default:  // TK_LMHEAD
        if (p.tied) {
            w0 = p.embed;
            esz = 2;
        } else {
            w0 = p.lm_head;
            s0 = p.lm_head_scale;
        }
        break;
    }
    g.K = K;
    g.esz = esz;
    g.RB = K * esz;
    const int gran = 16 / gcd16(g.RB);
    int rpc = p.stage_bytes / g.RB;
    rpc -= rpc % gran;
    g.rpc = rpc;
    g.R = d.r1 - d.r0;
    g.nck = (g.R + rpc - 1) / rpc;
    g.nchunks = g.nck * parts;
    g.base0 = static_cast<const uint8_t *>(w0) + (size_t)d.r0 * g.RB;
    g.base1 = w1 ? static_cast<const uint8_t *>(w1) + (size_t)d.r0 * g.RB : nullptr;
    g.scale0 = s0 ? s0 + d.r0 : nullptr;
    g.scale1 = s1 ? s1 + d.r0 : nullptr;
    return g;
}

// ------------------------------------------------------------------ producer
// Lane 0 of the producer warp streams every chunk of every task of this SM's
// queue into the ring.  Returns the number of chunks issued.
__device__ void producer_loop(const KParams &p, const SmemLayout &s, int qb, int qe)
{
    const uint64_t pol_w = evict_first_policy();  // weights: streamed once per step
    const int NS = p.ring_stages;
    uint32_t k = 0;  // chunks issued
    volatile int *abort_flag = s.flags;
    bool stop = false;
    for (int ti = qb; ti < qe && !stop; ++ti) {
        const TaskDesc d = p.tasks[ti];
        const Geom g = task_geom(p, d);
        for (int i = 0; i < g.nchunks; ++i, ++k) {
            const int st = k % NS;
            if (k >= (uint32_t)NS) {
                const uint32_t par = ((k / NS) - 1) & 1;
                uint32_t it = 0;
                uint64_t t0 = 0;
                while (!mbar_try_wait(&s.empty[st], par)) {
                    if (it == 0)
                        t0 = gtimer();
                    if ((++it & 255) == 0) {
                        if (*abort_flag || gtimer() - t0 > p.timeout_ns * 4 ||
                            it > (1u << 30)) {
                            stop = true;
                            break;
                        }
                    }
                }
                if (stop)
                    break;
            }
            uint8_t *dst = s.ring + (size_t)st * p.stage_bytes;
            if (d.kind == TK_ATTN) {
                const int a = g.pa + i * g.P;
                const int b = min(a + g.P, g.pb);
                const uint32_t nb = (uint32_t)(b - a) * p.head_dim * 2;
                mbar_arrive_expect_tx(&s.full[st], 2 * nb);
                bulk_g2s_nohint(dst, g.kb + (size_t)a * p.head_dim * 2, nb, &s.full[st]);
                bulk_g2s_nohint(dst + (size_t)g.P * p.head_dim * 2,
                                g.vb + (size_t)a * p.head_dim * 2, nb, &s.full[st]);
            } else {
                const int part = i / g.nck, c = i % g.nck;
                const int r = c * g.rpc;
                const int nr = min(g.rpc, g.R - r);
                const uint32_t nb = (uint32_t)nr * g.RB;
                const uint8_t *src = (part ? g.base1 : g.base0) + (size_t)r * g.RB;
                mbar_arrive_expect_tx(&s.full[st], nb);
                bulk_g2s(dst, src, nb, &s.full[st], pol_w);
            }
        }
    }
    // Drain: wait (bounded) for the copies still in flight so that no bulk
    // copy writes into shared memory after this CTA has exited.
    const uint32_t first = k > (uint32_t)NS ? k - NS : 0;
    for (uint32_t j = first; j < k; ++j) {
        const int st = j % NS;
        const uint32_t par = (j / NS) & 1;
        uint32_t it = 0;
        const uint64_t t1 = gtimer();
        while (!mbar_try_wait(&s.full[st], par)) {
            if ((++it & 255) == 0 && (gtimer() - t1 > p.timeout_ns || it > (1u << 30)))
                break;
        }
    }
}

// ------------------------------------------------------------------ consumers
struct CState {
    uint32_t k;      // chunks consumed
    bool aborted;
};

// Waits (all lanes of a warp together) until ring stage for chunk k is full.
__device__ __forceinline__ bool wait_full(const KParams &p, const SmemLayout &s, uint32_t k)
{
    const int st = k % p.ring_stages;
    const uint32_t par = (k / p.ring_stages) & 1;
    volatile int *abort_flag = s.flags;
    uint32_t it = 0;
    uint64_t t0 = 0;
    while (true) {
        const bool ok = mbar_try_wait(&s.full[st], par);
        if (__all_sync(0xffffffffu, ok))
            return true;
        if (it == 0)
            t0 = gtimer();
        if ((++it & 63) == 0) {
            const bool give_up = *abort_flag != 0 || gtimer() - t0 > p.timeout_ns ||
                                 it > (1u << 28);
            if (__any_sync(0xffffffffu, give_up))
                return false;
        }
    }
}

__device__ __forceinline__ void release_stage(const KParams &p, const SmemLayout &s,
                                              uint32_t k, int lane)
{
    __syncwarp();
    if (lane == 0)
        mbar_arrive(&s.empty[k % p.ring_stages]);
}

__device__ void record_error(const KParams &p, uint32_t code, int task, int ctr, uint32_t seen,
                             uint32_t target)
{
    if (atomicCAS(&p.err->code, 0u, code) == 0u) {
        p.err->task = task;
        p.err->counter = ctr;
        p.err->sm = blockIdx.x;
        p.err->seen = seen;
        p.err->target = target;
        __threadfence();
    }
}

// Counter wait by consumer thread 0; returns false on timeout / abort.
__device__ bool wait_counter(const KParams &p, const TaskDesc &d, int ti)
{
    if (d.wait_ctr < 0)
        return true;
    const uint32_t target = p.epoch * d.wait_total + d.wait_count;
    const uint32_t *ctr = p.counters + d.wait_ctr;
    const uint64_t t0 = gtimer();
    uint32_t v = 0;
    for (uint32_t it = 0;; ++it) {
        v = ld_acquire(ctr);
        if ((int32_t)(v - target) >= 0)
            return true;
        if ((it & 31) == 31) {
            if (ld_relaxed(&p.err->code) != 0u)
                return false;
            if (gtimer() - t0 > p.timeout_ns || it > (1u << 28)) {
                record_error(p, 1u, ti, d.wait_ctr, v, target);
                return false;
            }
        }
    }
}

// Block-wide sum over the 256 consumer threads (uses s.scr).
__device__ float block_sum(float v, const SmemLayout &s, int tid)
{
    v = warp_sum(v);
    if ((tid & 31) == 0)
        s.scr[tid >> 5] = v;
    consumer_bar();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w)
        t += s.scr[w];
    consumer_bar();
    return t;
}

// vec[i] = g_i * x_i / sqrt(mean x^2 + eps), x from L2 (fp32) or the
// embedding row (bf16).
__device__ void rmsnorm_prologue(const KParams &p, const SmemLayout &s, const float *x_f32,
                                 const uint16_t *x_bf16, const uint16_t *gain, int tid)
{
    const int n = p.hidden;
    float ss = 0.f;
    for (int i = tid; i < n; i += kConsumerThreads) {
        const float v = x_f32 ? __ldcg(x_f32 + i) : bf16_to_f(__ldg(x_bf16 + i));
        s.vec[i] = v;
        ss = fmaf(v, v, ss);
    }
    const float tot = block_sum(ss, s, tid);
    const float inv = rsqrtf(tot / (float)n + p.rms_eps);
    for (int i = tid; i < n; i += kConsumerThreads)
        s.vec[i] = bf16_to_f(__ldg(gain + i)) * (s.vec[i] * inv);
    consumer_bar();
}

// GEMV over a task's chunks.  Each warp owns vectors [vb, ve) of every row;
// lane l handles vb + l + 32 i.  Per-warp row sums go to red[w][row].
template <int ESZ, int VB>
__device__ bool gemv_task(const KParams &p, const SmemLayout &s, const Geom &g, CState &cs,
                          int warp, int lane)
{
    constexpr int E = VB / ESZ;
    constexpr int NI = 48 / E;
    const int NV = g.RB / VB;
    const int VPW = (NV + kConsumerWarps - 1) / kConsumerWarps;
    const int vb = warp * VPW;
    const int ve = min(vb + VPW, NV);
    float xr[NI][E];
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        const int v = vb + lane + 32 * i;
#pragma unroll
        for (int e = 0; e < E; ++e)
            xr[i][e] = (v < ve) ? s.vec[v * E + e] : 0.f;
    }
    float *red = s.red + warp * kMaxTaskRows;
    for (int i = 0; i < g.nchunks; ++i) {
        if (!wait_full(p, s, cs.k))
            return false;
        const uint8_t *stage = s.ring + (size_t)(cs.k % p.ring_stages) * p.stage_bytes;
        const int part = i / g.nck, c = i % g.nck;
        const int r = c * g.rpc;
        const int nr = min(g.rpc, g.R - r);
        const int rowbase = part * g.R + r;
        int j = 0;
        for (; j + 1 < nr; j += 2) {
            const uint8_t *row0 = stage + (size_t)j * g.RB;
            const uint8_t *row1 = row0 + g.RB;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int t = 0; t < NI; ++t) {
                const int v = vb + lane + 32 * t;
                if (v < ve) {
                    a0 = vdot<ESZ, VB>(row0 + (size_t)v * VB, xr[t], a0);
                    a1 = vdot<ESZ, VB>(row1 + (size_t)v * VB, xr[t], a1);
                }
            }
            a0 = warp_sum(a0);
            a1 = warp_sum(a1);
            if (lane == 0) {
                red[rowbase + j] = a0;
                red[rowbase + j + 1] = a1;
            }
        }
        if (j < nr) {
            const uint8_t *row0 = stage + (size_t)j * g.RB;
            float a0 = 0.f;
#pragma unroll
            for (int t = 0; t < NI; ++t) {
                const int v = vb + lane + 32 * t;
                if (v < ve)
                    a0 = vdot<ESZ, VB>(row0 + (size_t)v * VB, xr[t], a0);
            }
            a0 = warp_sum(a0);
            if (lane == 0)
                red[rowbase + j] = a0;
        }
        release_stage(p, s, cs.k, lane);
        ++cs.k;
    }
    return true;
}

__device__ bool run_gemv(const KParams &p, const SmemLayout &s, const Geom &g, CState &cs,
                         int warp, int lane)
{
    const int vbytes = (g.RB % 16 == 0) ? 16 : ((g.RB % 8 == 0) ? 8 : 4);
    if (g.esz == 2) {
        if (vbytes == 16)
            return gemv_task<2, 16>(p, s, g, cs, warp, lane);
        if (vbytes == 8)
            return gemv_task<2, 8>(p, s, g, cs, warp, lane);
        return gemv_task<2, 4>(p, s, g, cs, warp, lane);
    }
    if (vbytes == 16)
        return gemv_task<1, 16>(p, s, g, cs, warp, lane);
    if (vbytes == 8)
        return gemv_task<1, 8>(p, s, g, cs, warp, lane);
    return gemv_task<1, 4>(p, s, g, cs, warp, lane);
}

// Row sum over the 8 warps' partials for output row t of the task.
__device__ __forceinline__ float row_total(const SmemLayout &s, int t)
{
    float y = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w)
        y += s.red[w * kMaxTaskRows + t];
    return y;
}

__device__ __forceinline__ float row_scale(const uint16_t *scale, int t)
{
    return scale ? fp16_to_f(__ldg(scale + t)) : 1.f;
}

// RoPE (HF rotate_half) on a head vector in shared memory at position pos;
// angles in double precision: a = pos * theta^(-2i/hd).
__device__ void rope_smem(float *v, int hd, int pos, float theta, int i)
{
    const int half = hd / 2;
    if (i < half) {
        const double w = exp2(-(2.0 * i / hd) * log2((double)theta));
        double sn, cs;
        sincos((double)pos * w, &sn, &cs);
        const float c = (float)cs, sgn = (float)sn;
        const float x0 = v[i], x1 = v[i + half];
        v[i] = x0 * c - x1 * sgn;
        v[i + half] = x1 * c + x0 * sgn;
    }
}

// Split-K attention tile for KV head g and chunk c (flash-decoding partial):
// writes (m, l, o[hd]) per query head of the group, unnormalised.
__device__ bool attn_task(const KParams &p, const SmemLayout &s, const TaskDesc &d,
                          const Geom &g, CState &cs, int tid, int warp, int lane)
{
    const int l = d.layer, gi = d.r0, c = d.r1;
    const int hd = p.head_dim, G = p.group, nh = p.n_heads, nkv = p.n_kv_heads;
    const int lph = p.att_lph, E = p.att_e;
    float *qs = s.vec;                       // [G][hd], RoPE'd and pre-scaled
    float *kn = qs + G * hd;                 // [hd] new K row (bf16 value)
    float *vn = kn + hd;                     // [hd] new V row (bf16 value)
    float *ws = vn + hd;                     // [8][G][hd + 2] per-warp partials
    const float *qkv = p.qkv + (size_t)l * p.qkv_rows;
    if (g.j1 <= g.j0)
        return true;  // empty chunk: nothing to write, the combine skips it
    // prologue: load q (G heads), k, v of this KV head; RoPE q and k
    for (int i = tid; i < G * hd; i += kConsumerThreads)
        qs[i] = __ldcg(qkv + (size_t)gi * G * hd + i);
    for (int i = tid; i < hd; i += kConsumerThreads) {
        kn[i] = __ldcg(qkv + (size_t)nh * hd + (size_t)gi * hd + i);
        vn[i] = __ldcg(qkv + (size_t)(nh + nkv) * hd + (size_t)gi * hd + i);
    }
    consumer_bar();
    for (int i = tid; i < (G + 1) * (hd / 2); i += kConsumerThreads) {
        const int hh = i / (hd / 2), e = i % (hd / 2);
        rope_smem(hh < G ? qs + hh * hd : kn, hd, p.pos, p.rope_theta, e);
    }
    consumer_bar();
    const float scale = rsqrtf((float)hd);
    for (int i = tid; i < G * hd; i += kConsumerThreads)
        qs[i] *= scale;
    for (int i = tid; i < hd; i += kConsumerThreads) {
        const uint16_t kb = f_to_bf16(kn[i]), vb = f_to_bf16(vn[i]);
        kn[i] = bf16_to_f(kb);
        vn[i] = bf16_to_f(vb);
        if (c == 0) {
            const size_t blk = (size_t)p.max_ctx * hd;
            p.kv[(((size_t)l * 2 + 0) * nkv + gi) * blk + (size_t)p.pos * hd + i] = kb;
            p.kv[(((size_t)l * 2 + 1) * nkv + gi) * blk + (size_t)p.pos * hd + i] = vb;
        }
    }
    consumer_bar();
    // lane layout: head jh = lane / lph (within the group), elements
    // [e0, e0 + E) of that head
    const int jh = lane / lph;
    const int e0 = (lane % lph) * E;
    const bool active = jh < G;
    float q[32], o[32];
    float m = -INFINITY, lsum = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        q[e] = (active && e < E) ? qs[jh * hd + e0 + e] : 0.f;
        o[e] = 0.f;
    }
    auto visit = [&](const float *krow_f, const uint16_t *krow_b, const float *vrow_f,
                     const uint16_t *vrow_b) {
        float sc = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if (e < E)
                sc = fmaf(q[e], krow_b ? bf16_to_f(krow_b[e0 + e]) : krow_f[e0 + e], sc);
        for (int off = lph >> 1; off > 0; off >>= 1)
            sc += __shfl_xor_sync(0xffffffffu, sc, off);
        const float mn = fmaxf(m, sc);
        const float corr = __expf(m - mn);
        const float pr = __expf(sc - mn);
        lsum = lsum * corr + pr;
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if (e < E)
                o[e] = o[e] * corr + pr * (vrow_b ? bf16_to_f(vrow_b[e0 + e]) : vrow_f[e0 + e]);
        m = mn;
    };
    bool fail = false;
    for (int i = 0; i < g.nchunks; ++i) {
        if (!wait_full(p, s, cs.k)) {
            fail = true;
            break;
        }
        const uint8_t *stage = s.ring + (size_t)(cs.k % p.ring_stages) * p.stage_bytes;
        const uint16_t *Ks = reinterpret_cast<const uint16_t *>(stage);
        const uint16_t *Vs = reinterpret_cast<const uint16_t *>(stage + (size_t)g.P * hd * 2);
        const int a = g.pa + i * g.P;
        const int n = min(g.P, g.pb - a);
        for (int j = warp; j < n; j += kConsumerWarps)
            visit(nullptr, Ks + (size_t)j * hd, nullptr, Vs + (size_t)j * hd);
        release_stage(p, s, cs.k, lane);
        ++cs.k;
    }
    if (fail && lane == 0)
        s.flags[0] = 1;
    consumer_bar();
    if (*reinterpret_cast<volatile int *>(s.flags))
        return false;
    if (g.j0 <= p.pos && p.pos < g.j1 && warp == 0)
        visit(kn, nullptr, vn, nullptr);
    // per-warp state -> ws[w][jh][hd + 2]
    float *mine = ws + (size_t)warp * G * (hd + 2);
    if (active) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if (e < E)
                mine[jh * (hd + 2) + 2 + e0 + e] = o[e];
        if (lane % lph == 0) {
            mine[jh * (hd + 2) + 0] = m;
            mine[jh * (hd + 2) + 1] = lsum;
        }
    }
    consumer_bar();
    float *out = p.part + ((((size_t)l * nkv + gi) * p.attn_splits + c) * G) * (hd + 2);
    for (int i = tid; i < G * hd; i += kConsumerThreads) {
        const int hh = i / hd, e = i % hd;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w)
            M = fmaxf(M, ws[((size_t)w * G + hh) * (hd + 2)]);
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float *pw = ws + ((size_t)w * G + hh) * (hd + 2);
            const float f = (pw[1] > 0.f) ? __expf(pw[0] - M) : 0.f;
            L = fmaf(pw[1], f, L);
            O = fmaf(pw[2 + e], f, O);
        }
        out[(size_t)hh * (hd + 2) + 2 + e] = O;
        if (e == 0) {
            out[(size_t)hh * (hd + 2) + 0] = M;
            out[(size_t)hh * (hd + 2) + 1] = L;
        }
    }
    return true;
}

// O-projection prologue: combine the split-K partials of every head into
// the attention output vec[h * hd + e] = sum_c w_c o_c[e] / L.
__device__ void combine_prologue(const KParams &p, const SmemLayout &s, int l, int tid)
{
    const int hd = p.head_dim, nh = p.n_heads, G = p.group, C = p.attn_splits;
    const int n = p.pos + 1;
    const int chunk = (n + C - 1) / C;
    const int nne = (n + chunk - 1) / chunk;  // non-empty splits
    float *wts = s.vec + (size_t)nh * hd;     // [nh][C]
    const float *part = p.part + (size_t)l * p.n_kv_heads * C * G * (hd + 2);
    for (int h = tid; h < nh; h += kConsumerThreads) {
        const int gi = h / G, jh = h % G;
        float M = -INFINITY;
        for (int c = 0; c < nne; ++c)
            M = fmaxf(M, __ldcg(part + (((size_t)gi * C + c) * G + jh) * (hd + 2)));
        float L = 0.f;
        for (int c = 0; c < nne; ++c) {
            const float *pc = part + (((size_t)gi * C + c) * G + jh) * (hd + 2);
            const float f = __expf(__ldcg(pc) - M);
            wts[(size_t)h * C + c] = f;
            L = fmaf(__ldcg(pc + 1), f, L);
        }
        const float inv = 1.f / L;
        for (int c = 0; c < nne; ++c)
            wts[(size_t)h * C + c] *= inv;
    }
    consumer_bar();
    for (int i = tid; i < nh * hd; i += kConsumerThreads) {
        const int h = i / hd, e = i % hd;
        const int gi = h / G, jh = h % G;
        float acc = 0.f;
        for (int c = 0; c < nne; ++c)
            acc = fmaf(wts[(size_t)h * C + c],
                       __ldcg(part + (((size_t)gi * C + c) * G + jh) * (hd + 2) + 2 + e), acc);
        s.vec[i] = acc;
    }
    consumer_bar();
}

__device__ __forceinline__ unsigned long long argmax_key(float v, int idx)
{
    v = v + 0.0f;  // -0 -> +0
    uint32_t u = __float_as_uint(v);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)u << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)idx);
}

__device__ int resolve_token(const KParams &p)
{
    int t = p.token;
    if (t < 0) {
        const unsigned long long key = __ldcg(p.argkey + (p.parity ^ 1));
        t = (int)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
    }
    if (t < 0 || t >= p.vocab) {
        record_error(p, 3u, -1, -1, (uint32_t)t, 0u);
        t = 0;
    }
    return t;
}

// ------------------------------------------------------------------- kernel
__global__ void __launch_bounds__(kThreads, 1) amk_decode_kernel(const __grid_constant__ KParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const SmemLayout s = smem_layout(smem_raw, p);
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int qb = p.queue_off[blockIdx.x], qe = p.queue_off[blockIdx.x + 1];

    if (tid == 0) {
        for (int i = 0; i < p.ring_stages; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], kConsumerWarps);
        }
        // a failed earlier step poisons the device state: do no work until the
        // host resets it (the counters no longer match the epoch)
        s.flags[0] = ld_relaxed(&p.err->code) != 0u ? 1 : 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();
    if (s.flags[0])
        return;

    if (warp == kConsumerWarps) {
        if (lane == 0)
            producer_loop(p, s, qb, qe);
        return;
    }

    CState cs{0u, false};
    int token = -1;
    for (int ti = qb; ti < qe; ++ti) {
        const TaskDesc d = p.tasks[ti];
        if (tid == 0) {
            if (!wait_counter(p, d, ti))
                s.flags[0] = 1;
        }
        consumer_bar();
        if (*reinterpret_cast<volatile int *>(s.flags))
            break;
        const Geom g = task_geom(p, d);
        const int l = d.layer;
        bool ok = true;
        if (d.kind == TK_ATTN) {
            ok = attn_task(p, s, d, g, cs, tid, warp, lane);
        } else {
            // prologue -> s.vec
            if (d.kind == TK_QKV) {
                if (l == 0) {
                    if (token < 0)
                        token = resolve_token(p);
                    rmsnorm_prologue(p, s, nullptr, p.embed + (size_t)token * p.hidden,
                                     p.layers[0].attn_norm, tid);
                } else {
                    rmsnorm_prologue(p, s, p.xout + (size_t)(l - 1) * p.hidden, nullptr,
                                     p.layers[l].attn_norm, tid);
                }
            } else if (d.kind == TK_OPROJ) {
                combine_prologue(p, s, l, tid);
            } else if (d.kind == TK_GATEUP) {
                rmsnorm_prologue(p, s, p.xmid + (size_t)l * p.hidden, nullptr,
                                 p.layers[l].ffn_norm, tid);
            } else if (d.kind == TK_DOWN) {
                const float *a = p.act + (size_t)l * p.ffn;
                for (int i = tid; i < p.ffn; i += kConsumerThreads)
                    s.vec[i] = __ldcg(a + i);
                consumer_bar();
            } else {  // TK_LMHEAD
                rmsnorm_prologue(p, s, p.xout + (size_t)(p.n_layers - 1) * p.hidden, nullptr,
                                 p.final_norm, tid);
            }
            ok = run_gemv(p, s, g, cs, warp, lane);
            if (!ok && lane == 0) {
                record_error(p, 2u, ti, -1, 0u, 0u);
                s.flags[0] = 1;
            }
            consumer_bar();
            ok = *reinterpret_cast<volatile int *>(s.flags) == 0;
            if (ok) {
                // epilogue: thread t finalises output row r0 + t
                if (d.kind == TK_QKV) {
                    const int off = d.mat == 0 ? 0
                                    : d.mat == 1 ? p.n_heads * p.head_dim
                                                 : (p.n_heads + p.n_kv_heads) * p.head_dim;
                    float *out = p.qkv + (size_t)l * p.qkv_rows + off + d.r0;
                    for (int t = tid; t < g.R; t += kConsumerThreads)
                        out[t] = row_total(s, t) * row_scale(g.scale0, t);
                } else if (d.kind == TK_OPROJ) {
                    for (int t = tid; t < g.R; t += kConsumerThreads) {
                        const int r = d.r0 + t;
                        float base;
                        if (l == 0) {
                            if (token < 0)
                                token = resolve_token(p);
                            base = bf16_to_f(__ldg(p.embed + (size_t)token * p.hidden + r));
                        } else {
                            base = __ldcg(p.xout + (size_t)(l - 1) * p.hidden + r);
                        }
                        p.xmid[(size_t)l * p.hidden + r] =
                            base + row_total(s, t) * row_scale(g.scale0, t);
                    }
                } else if (d.kind == TK_GATEUP) {
                    for (int t = tid; t < g.R; t += kConsumerThreads) {
                        const float gt = row_total(s, t) * row_scale(g.scale0, t);
                        const float up = row_total(s, g.R + t) * row_scale(g.scale1, t);
                        const float silu = gt / (1.f + __expf(-gt));
                        p.act[(size_t)l * p.ffn + d.r0 + t] = silu * up;
                    }
                } else if (d.kind == TK_DOWN) {
                    for (int t = tid; t < g.R; t += kConsumerThreads) {
                        const int r = d.r0 + t;
                        p.xout[(size_t)l * p.hidden + r] =
                            __ldcg(p.xmid + (size_t)l * p.hidden + r) +
                            row_total(s, t) * row_scale(g.scale0, t);
                    }
                } else {  // TK_LMHEAD
                    unsigned long long best = 0ull;
                    for (int t = tid; t < g.R; t += kConsumerThreads) {
                        const float y = row_total(s, t) * row_scale(g.scale0, t);
                        p.logits[d.r0 + t] = y;
                        const unsigned long long kk = argmax_key(y, d.r0 + t);
                        best = kk > best ? kk : best;
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
                        best = other > best ? other : best;
                    }
                    unsigned long long *sk = reinterpret_cast<unsigned long long *>(s.scr);
                    if (lane == 0)
                        sk[warp] = best;
                    consumer_bar();
                    if (tid == 0) {
                        unsigned long long b = 0ull;
                        for (int w = 0; w < kConsumerWarps; ++w)
                            b = sk[w] > b ? sk[w] : b;
                        atomicMax(p.argkey + p.parity, b);
                        if (d.flags & TF_RESET_ARGKEY)
                            p.argkey[p.parity ^ 1] = 0ull;
                    }
                }
            }
        }
        if (!ok)
            s.flags[0] = 1;
        consumer_bar();
        if (*reinterpret_cast<volatile int *>(s.flags))
            break;
        if (tid == 0 && d.signal_ctr >= 0 && ti != p.skip_signal_task) {
            __threadfence();
            red_release_add(p.counters + d.signal_ctr, 1u);
        }
    }
    // On abort the producer notices the flag, drains its copies and returns.
}

}  // namespace

// Host-visible launch helpers -------------------------------------------------
extern "C" int amk_kernel_smem_bytes(int ring_stages, int stage_bytes, int vec_floats)
{
    return ring_stages * stage_bytes + vec_floats * 4 + kConsumerWarps * kMaxTaskRows * 4 +
           2 * kMaxStages * 8 + 16 * 4 + 64 * 4;
}

extern "C" cudaError_t amk_kernel_configure(int smem_bytes)
{
    return cudaFuncSetAttribute(amk_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                smem_bytes);
}

extern "C" cudaError_t amk_kernel_occupancy(int smem_bytes, int *blocks_per_sm)
{
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, amk_decode_kernel,
                                                         kThreads, smem_bytes);
}

extern "C" cudaError_t amk_kernel_launch(const KParams *p, int n_ctas, int smem_bytes,
                                         cudaStream_t stream)
{
    void *args[] = {const_cast<KParams *>(p)};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(amk_decode_kernel),
                                       dim3(n_ctas), dim3(kThreads), args, (size_t)smem_bytes,
                                       stream);
}

}  // namespace amk
