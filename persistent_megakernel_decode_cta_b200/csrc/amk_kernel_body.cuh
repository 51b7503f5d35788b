// amk_kernel_body.cuh -- the persistent decode megakernel for sm_100a.
//
// Device code only, included by the instance files amk_kernel_inst_*.cu
// (each compiles some of the kernel's template instances, so that the
// instances build in parallel); amk_kernel.cu holds the launch helpers.
//
// One launch = one forward pass = one token ("RightNow-AI/AutoMegaKernel"
// README, opening summary).  One CTA per SM walks its own queue of tasks in a
// global topological order: wait for the inputs -> run the task -> hand the
// outputs on (gist.science technical summary, "Methodologie", layer 0;
// paperfeed review, "How it works").  The pages wait on counters with
// statically known thresholds (README, "Deadlock-free by construction"); by
// default this kernel waits on the data itself instead: every vector a level
// hands to the next is made of flagged words (value + step tag in one word,
// see fw_st / fw32_st), and a task's poll of the words it reads is its wait.
// The counter protocol remains for the fused FFN level and on request.
// Weights of upcoming tasks are prefetched while the current one computes
// (README, "Why a megakernel").
//
// B200 design (not the pages' sm_80..sm_120 design):
//  * 384 threads per CTA in three warpgroups.  The producer warpgroup gives
//    up registers (setmaxnreg) and one lane walks the SM's queue AHEAD of the
//    consumers, copying each task's weight rows (or KV-cache rows) into a
//    ring of shared-memory stages with cp.async.bulk (TMA bulk copies) that
//    complete on per-stage mbarriers.  Weights never depend on activations,
//    so the copies run ahead across counter waits.
//  * Two consumer warpgroups (8 warps) take the freed registers.  They poll
//    the flagged words of the task's inputs (or, with level counters, spin
//    on the task's counter with ld.acquire.gpu; both with a time limit),
//    build the task's input vector in shared memory (RMSNorm / attention
//    output prologues), run the GEMV from the ring -- each warp owns a
//    K-slice whose activations sit in registers -- reduce with warp
//    shuffles, and apply the fused epilogue (RoPE + KV append, SwiGLU,
//    residual add, argmax), whose flagged stores are the task's signal (with
//    level counters: a red.release.gpu on the task's counter).
//  * Task records carry host-resolved pointers and are prefetched one task
//    ahead, so no task boundary waits on a dependent global load.
//  * Every wait is bounded (globaltimer + iteration cap); on expiry the CTA
//    records the failure, drains its own TMA copies and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#pragma once
#include "amk_internal.h"

namespace amk {
namespace {

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Non-blocking test of the same phase completion (never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void bulk_g2s_nohint(uint32_t dst, const void *src, uint32_t bytes,
                                                uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
// Tiled 2-D TMA load of the box at (x, y) of the tensor map at tmap (a
// generic address of a 64-byte aligned CUtensorMap in global memory) into
// shared memory, completing on the mbarrier bar.  No multicast.  x (the
// innermost coordinate) times the element size is a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *tmap, int x, int y,
                                            uint32_t bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(tmap), "r"(x), "r"(y), "r"(bar), "l"(policy)
        : "memory");
}
// Acquire fence of the tensor-map proxy on the 128-byte map at tmap (global
// memory): a map written through the generic proxy (or by a host copy) before
// this point is the one the next tensor copies through it read.
__device__ __forceinline__ void tmap_acquire(const void *tmap)
{
    asm volatile("fence.proxy.tensormap::generic.acquire.sys [%0], 128;" ::"l"(tmap) : "memory");
}
// Fetches [src, src + bytes) from HBM into L2 only (no shared-memory
// destination, no completion tracking).
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
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
// Flagged words carry a value from one level to the next: the fp32 value in
// the low half and the tag of the step that wrote it in the high half of one
// aligned 64-bit word, stored and loaded as single relaxed accesses at GPU
// scope (each is single-copy atomic).  A reader that finds its step's tag
// holds that step's value, so the writer issues no fence before its readers
// may go on, and a reader's poll of the data is its whole wait.
__device__ __forceinline__ void fw_st(uint64_t *a, float v, uint32_t tag)
{
    const uint64_t w = ((uint64_t)tag << 32) | (uint64_t)__float_as_uint(v);
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(a), "l"(w) : "memory");
}
__device__ __forceinline__ uint64_t fw_ld(const uint64_t *a)
{
    uint64_t w;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(w) : "l"(a) : "memory");
    return w;
}
// two consecutive words (16-byte aligned), each loaded as its own access
__device__ __forceinline__ void fw_ld2(const uint64_t *a, uint64_t &x, uint64_t &y)
{
    asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];"
                 : "=l"(x), "=l"(y)
                 : "l"(a)
                 : "memory");
}
__device__ __forceinline__ float fw_val(uint64_t w) { return __uint_as_float((uint32_t)w); }
__device__ __forceinline__ bool fw_ok(uint64_t w, uint32_t tag) { return (uint32_t)(w >> 32) == tag; }
// The SwiGLU activations, read by every SM in full for the down projection,
// are 32-bit flagged words instead (half the bytes to load and to poll): the
// fp32 value with its 8 low mantissa bits replaced by an 8-bit step tag in
// 1 .. 255 (consecutive steps differ; cleared memory never matches, and
// every such word is rewritten every step, so a stale one is one step old
// and never passes), so a value keeps 15 mantissa bits, rounded to nearest
// (a relative error of at most 2^-16) -- finer than the int16 steps the
// int8 / int4 GEMV takes its activations in, and than the bf16 weights they
// multiply.
__device__ __forceinline__ uint32_t fw8_tag(uint32_t tag) { return tag % 255u + 1u; }
__device__ __forceinline__ void fw32_st(uint32_t *a, float v, uint32_t t8)
{
    // round to the nearest 15-bit mantissa (half away from zero: the add
    // carries into the exponent when the mantissa overflows), then the tag;
    // truncating instead biased every value toward zero, and the down
    // projection's long sums added that bias up
    const uint32_t w = ((__float_as_uint(v) + 0x80u) & ~0xffu) | t8;
    asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(a), "r"(w) : "memory");
}
// four consecutive words (16-byte aligned), each loaded as its own access
__device__ __forceinline__ void fw32_ld4(const uint32_t *a, uint32_t (&w)[4])
{
    asm volatile("ld.relaxed.gpu.global.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                 : "l"(a)
                 : "memory");
}
__device__ __forceinline__ void fw32_ld2(const uint32_t *a, uint32_t (&w)[2])
{
    asm volatile("ld.relaxed.gpu.global.v2.b32 {%0, %1}, [%2];"
                 : "=r"(w[0]), "=r"(w[1])
                 : "l"(a)
                 : "memory");
}
__device__ __forceinline__ float fw32_val(uint32_t w) { return __uint_as_float(w & ~0xffu); }
__device__ __forceinline__ bool fw32_ok(uint32_t w, uint32_t t8) { return (w & 0xffu) == t8; }
// The residual after a fused FFN level is held in fixed point (value * 2^32
// in an int64): integer addition is associative, so the FFN slices' partial
// down projections add up to the same bits in any order.  |value| < 2^31.
__device__ __forceinline__ long long to_fix(float v) { return __float2ll_rn(v * 4294967296.0f); }
__device__ __forceinline__ float from_fix(long long a)
{
    return (float)((double)a * (1.0 / 4294967296.0));
}
__device__ __forceinline__ void red_add_fix(long long *p, long long v)
{
    asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
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
template <int N>
__device__ __forceinline__ void setmaxnreg_inc()
{
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec()
{
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Explicit shared-memory accesses by 32-bit shared address, so the hot
// loops use ld.shared/st.shared.  Ordering against the ring's TMA writes
// comes from the mbarrier waits (asm volatile with a memory clobber).
__device__ __forceinline__ uint4 lds128(uint32_t a)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a)
{
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a)
{
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ void stsf(uint32_t a, float v)
{
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v));
}

// ------------------------------------------------------------- number formats
__device__ __forceinline__ float bf16_to_f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }
__device__ __forceinline__ uint16_t f_to_bf16(float f)
{
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
__device__ __forceinline__ float fp16_to_f(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// Packed pairs of floats (f32x2 arithmetic: one instruction per two lanes'
// worth of work).
typedef unsigned long long f2_t;
__device__ __forceinline__ f2_t pk2(float a, float b)
{
    f2_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float sum2(f2_t r)
{
    float a, b;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
    return a + b;
}
__device__ __forceinline__ f2_t ffma2(f2_t a, f2_t b, f2_t c)
{
    f2_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ f2_t fadd2(f2_t a, f2_t b)
{
    f2_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// two bf16 in a word -> (low, high) as a float pair
__device__ __forceinline__ f2_t bf2(uint32_t w)
{
    f2_t r;
    asm("{\n\t.reg .b32 lo, hi;\n\tshl.b32 lo, %1, 16;\n\tand.b32 hi, %1, 0xffff0000;\n\t"
        "mov.b64 %0, {lo, hi};\n\t}"
        : "=l"(r)
        : "r"(w));
    return r;
}
// four int8 in a word -> two float pairs, exactly: 0x4B000000 | (q + 128) is
// the float 2^23 + q + 128, and the pair subtraction removes the offset
__device__ __forceinline__ void i8x4(uint32_t w, f2_t &lo, f2_t &hi)
{
    const uint32_t b = w ^ 0x80808080u;
    const f2_t off = pk2(-8388736.0f, -8388736.0f);
    lo = fadd2(pk2(__uint_as_float(__byte_perm(b, 0x4B000000u, 0x7440)),
                   __uint_as_float(__byte_perm(b, 0x4B000000u, 0x7441))), off);
    hi = fadd2(pk2(__uint_as_float(__byte_perm(b, 0x4B000000u, 0x7442)),
                   __uint_as_float(__byte_perm(b, 0x4B000000u, 0x7443))), off);
}

// A weight vector of VB bytes held in registers.
template <int VB> struct WVec;
template <> struct WVec<16> { uint32_t w[4]; };
template <> struct WVec<8> { uint32_t w[2]; };
template <> struct WVec<4> { uint32_t w[1]; };

template <int VB>
__device__ __forceinline__ WVec<VB> ldw(uint32_t a)
{
    WVec<VB> v;
    if constexpr (VB == 16) {
        const uint4 t = lds128(a);
        v.w[0] = t.x;
        v.w[1] = t.y;
        v.w[2] = t.z;
        v.w[3] = t.w;
    } else if constexpr (VB == 8) {
        const uint2 t = lds64(a);
        v.w[0] = t.x;
        v.w[1] = t.y;
    } else {
        v.w[0] = lds32(a);
    }
    return v;
}

// acc += (weights of v) . x over packed pairs; x holds VB/ESZ/2 float pairs
template <int ESZ, int VB>
__device__ __forceinline__ f2_t vdot2(const WVec<VB> &v, const f2_t *x, f2_t acc)
{
#pragma unroll
    for (int i = 0; i < VB / 4; ++i) {
        if constexpr (ESZ == 2) {
            acc = ffma2(bf2(v.w[i]), x[i], acc);
        } else {
            f2_t lo, hi;
            i8x4(v.w[i], lo, hi);
            acc = ffma2(lo, x[2 * i], acc);
            acc = ffma2(hi, x[2 * i + 1], acc);
        }
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
    uint64_t *full;       // [kMaxStages][kPieces]: stage st, piece pc at st * kPieces + pc
    uint64_t *empty;      // [kMaxStages]
    int *flags;           // [0] abort
    float *scr;           // 64 floats of reduction scratch
    unsigned long long *wacc;  // [2] per-task sums over warps (profiling)
    uint4 *pq;            // [kPieceQueue] producer's pieces in flight: (bar, parity, bytes, chunk)
    uint32_t ring_a, vec_a, red_a, full_a, empty_a;  // shared addresses
    uint32_t ptask_a, ctask_a;  // [2] staged task records of producer / consumers
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
    off += kMaxStages * kPieces * 8;
    s.empty = reinterpret_cast<uint64_t *>(base + off);
    off += kMaxStages * 8;
    s.flags = reinterpret_cast<int *>(base + off);
    off += 16 * 4;
    s.scr = reinterpret_cast<float *>(base + off);
    off += 64 * 4;
    s.wacc = reinterpret_cast<unsigned long long *>(base + off);
    off += 16;
    s.pq = reinterpret_cast<uint4 *>(base + off);
    off += kPieceQueue * 16;
    s.ptask_a = smem_u32(base + off);
    off += 2 * sizeof(TaskDesc);
    s.ctask_a = smem_u32(base + off);
    s.ring_a = smem_u32(s.ring);
    s.vec_a = smem_u32(s.vec);
    s.red_a = smem_u32(s.red);
    s.full_a = smem_u32(s.full);
    s.empty_a = smem_u32(s.empty);
    return s;
}

// Copies a task record into a shared-memory slot asynchronously (cp.async,
// six 16-byte pieces, one commit group), holding no registers; the issuing
// thread waits for it with stage_task_wait before anyone reads the slot.
__device__ __forceinline__ void stage_task(uint32_t slot, const TaskDesc *t)
{
    const uint8_t *src = reinterpret_cast<const uint8_t *>(t);
#pragma unroll
    for (int i = 0; i < (int)sizeof(TaskDesc) / 16; ++i)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(slot + 16 * i),
                     "l"(src + 16 * i)
                     : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void stage_task_wait()
{
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ TaskDesc read_staged(uint32_t slot)
{
    TaskDesc d;
    uint4 *dst = reinterpret_cast<uint4 *>(&d);
#pragma unroll
    for (int i = 0; i < (int)sizeof(TaskDesc) / 16; ++i)
        dst[i] = lds128(slot + 16 * i);
    return d;
}

// A GEMV's input vector in shared memory is padded by 16 bytes after every
// 128 (element i at vidx(i)): a lane reads its E-element pieces of the
// vector with 16-byte loads, and lanes 32 or 64 bytes apart would otherwise
// share banks (8 lanes of a wavefront into 2 or 4 bank groups); with the
// padding they fall into 8 distinct groups.
__device__ __forceinline__ int vidx(int i) { return i + ((i >> 5) << 2); }

// ------------------------------------------------------------- task geometry
// Both the producer and the consumers derive a task's chunk stream from its
// record with this function (no memory reads), so they agree on every chunk.
struct Geom {
    int nchunks;
    int ngu;  // chunks of the row-GEMV parts (all of them but a fused FFN's Wdown part)
    // GEMV tiles
    int K, esz, RB, rpc, R, nck;
    // fused FFN, Wdown part: the slice's columns in boxes of 16 bytes x BR rows;
    // chunk c covers rows [c rpc2, min(h, (c + 1) rpc2)), rpc2 a multiple of 256
    // or all of h
    int ncb, rpc2, nck2;
    int VB, KS, RG;  // vector bytes; warps split K into KS slices x RG row groups
    int ks_log2, rg_log2;
    // attention tiles
    int j0, j1, pa, pb, P;
};

__device__ __forceinline__ Geom task_geom(const KParams &p, const TaskDesc &d)
{
    Geom g{};
    if (d.kind == TK_ATTN) {
        const int c = d.r1;
        const int n = p.pos + 1;
        const int chunk = p.att_chunk;  // positions per chunk at this step
        g.j0 = c * chunk;
        g.j1 = min(g.j0 + chunk, n);
        if (g.j1 < g.j0)
            g.j1 = g.j0;
        g.pa = g.j0;
        g.pb = max(g.pa, min(g.j1, p.pos));
        g.P = p.att_P;
        g.nchunks = (g.pb - g.pa + g.P - 1) / g.P;
        return g;
    }
    // GEMV tiles: the chunk stream and warp layout come with the record
    // (the host computed them when it resolved the task)
    // bytes per weight: 2 (bf16), 1 (int8), 0 (packed int4 rows with their scales)
    int K = p.hidden, esz = p.quant == 1 ? 1 : p.quant == 2 ? 0 : 2;
    if (d.kind == TK_OPROJ)
        K = p.n_heads * p.head_dim;
    else if (d.kind == TK_DOWN)
        K = p.ffn;
    else if (d.kind == TK_LMHEAD && p.tied)
        esz = 2;
    g.K = K;
    g.esz = esz;
    g.RB = esz ? K * esz : q4_row_bytes(K);
    g.VB = (g.RB & 15) == 0 ? 16 : ((g.RB & 7) == 0 ? 8 : 4);
    g.R = d.r1 - d.r0;
    g.rpc = d.rpc;
    g.nck = d.nck;
    g.ngu = d.ngu;
    g.nchunks = d.nchunks;
    g.ncb = d.ncb;
    g.rpc2 = d.rpc2;
    g.nck2 = d.nck2;
    g.ks_log2 = d.ks_log2;
    g.rg_log2 = d.rg_log2;
    g.KS = 1 << d.ks_log2;
    g.RG = 1 << d.rg_log2;
    return g;
}

// ------------------------------------------------------------------ producer
// L2 lookahead (optional).  A task's byte stream is at most two contiguous
// regions (the rows of a GEMV tile, or of its gate and up halves; the K and
// V rows of an attention chunk range), copied into the ring in that order.
// While the ring is full -- typically while the consumers wait at a level
// boundary -- the producer walks a second cursor over the same streams and
// prefetches up to `lookahead` bytes past its copy cursor into L2, so that
// HBM keeps streaming and the ring refills from L2 once the consumers resume.
struct Lookahead {
    const uint8_t *a, *b;  // regions of the cursor's task
    uint32_t na, nb;
    uint32_t off;          // bytes of the current region already passed
    int ti;                // task of the cursor (qe: end of the queue)
    int part;              // 0: region a, 1: region b, 2: task exhausted
    uint64_t pos;          // stream position of the cursor
};

__device__ __forceinline__ void lookahead_load(const KParams &p, Lookahead &la)
{
    const uint8_t *rec = reinterpret_cast<const uint8_t *>(p.tasks + la.ti);
    TaskDesc d{};
    d.kind = (uint8_t)__ldg(reinterpret_cast<const uint32_t *>(rec));
    const int4 q = __ldg(reinterpret_cast<const int4 *>(rec + 16));  // ..., r0, r1
    const longlong2 w = __ldg(reinterpret_cast<const longlong2 *>(rec + 32));  // w0, w1
    d.r0 = q.z;
    d.r1 = q.w;
    // the geometry fields (the record's last 16 bytes)
    const int4 gq = __ldg(reinterpret_cast<const int4 *>(rec + 80));
    memcpy(reinterpret_cast<uint8_t *>(&d) + 80, &gq, 16);
    const Geom g = task_geom(p, d);
    const uint8_t *w0 = reinterpret_cast<const uint8_t *>(w.x);
    const uint8_t *w1 = reinterpret_cast<const uint8_t *>(w.y);
    if (d.kind == TK_ATTN) {
        const size_t o = (size_t)g.pa * p.head_dim * 2;
        la.a = w0 + o;
        la.b = w1 + o;
        la.na = la.nb = (uint32_t)(g.pb - g.pa) * p.head_dim * 2;
    } else {
        la.a = w0;
        la.b = w1;
        la.na = (uint32_t)g.R * g.RB;
        la.nb = g.nchunks > g.nck ? la.na : 0u;
    }
    la.part = 0;
    la.off = 0;
}

// Advances the cursor to stream position `hi`, prefetching the bytes at or
// past `lo` (the copy cursor: bytes before it are in the ring already).
__device__ __forceinline__ void lookahead_pump(const KParams &p, Lookahead &la, int qe,
                                               uint64_t lo, uint64_t hi)
{
    constexpr uint32_t kPiece = 32768;
    while (la.pos < hi && la.ti < qe) {
        if (la.part >= 2) {
            if (++la.ti >= qe)
                return;
            lookahead_load(p, la);
            continue;
        }
        const uint8_t *base = la.part ? la.b : la.a;
        const uint32_t n = la.part ? la.nb : la.na;
        if (la.off >= n) {
            ++la.part;
            la.off = 0;
            continue;
        }
        uint32_t piece = min(n - la.off, kPiece);
        if (la.pos < lo)  // already copied: skip without prefetching
            piece = (uint32_t)min((uint64_t)piece, lo - la.pos);
        else
            bulk_prefetch_l2(base + la.off, piece);
        la.off += piece;
        la.pos += piece;
    }
}

// Bulk-copy bytes in flight.  Copies the producer has issued wait in the
// SM's memory queues together with every other access of the SM, so the
// more there are, the longer each L2 hit, counter poll and release takes
// (on B200 an L2 hit goes from ~0.2 us idle to ~0.6 us with 64 KiB in
// flight per SM and ~1.2 us with 192 KiB, while 64 KiB already draws ~96 %
// of the stream bandwidth).  The producer therefore issues each chunk in
// pieces on their own mbarriers and keeps at most p.inflight bytes
// outstanding; the ring still fills completely while consumers wait.
struct Flight {
    uint32_t head, tail;  // queue positions (pieces issued: tail)
    uint32_t bytes;       // bytes of the queued pieces
};

// Drops completed pieces from the front of the queue, and every piece of
// a chunk below `done_below` (those are known complete: their stage has
// been consumed).
__device__ __forceinline__ void flight_retire(const SmemLayout &s, Flight &f, uint32_t done_below)
{
    while (f.head != f.tail) {
        const uint4 e = s.pq[f.head % kPieceQueue];
        if (e.w >= done_below && !mbar_test_wait(e.x, e.y))
            break;
        f.bytes -= e.z;
        ++f.head;
    }
}

// Waits (bounded) until `bytes` more fit under the cap; false on abort.
__device__ bool flight_reserve(const KParams &p, const SmemLayout &s, Flight &f, uint32_t bytes,
                               uint32_t done_below, uint64_t &prof_wait)
{
    flight_retire(s, f, done_below);
    volatile int *abort_flag = s.flags;
    uint32_t it = 0;
    uint64_t t0 = 0;
    while (f.head != f.tail && (f.bytes + bytes > p.inflight || f.tail - f.head >= kPieceQueue)) {
        const uint4 e = s.pq[f.head % kPieceQueue];
        if (mbar_try_wait(e.x, e.y)) {
            f.bytes -= e.z;
            ++f.head;
            continue;
        }
        if (it == 0)
            t0 = gtimer();
        if ((++it & 255) == 0 &&
            (*abort_flag || gtimer() - t0 > p.timeout_ns * 4 || it > (1u << 30)))
            return false;
    }
    if (p.prof && it)
        prof_wait += gtimer() - t0;
    return true;
}

__device__ __forceinline__ void flight_push(const SmemLayout &s, Flight &f, uint32_t bar,
                                            uint32_t par, uint32_t bytes, uint32_t chunk)
{
    s.pq[f.tail % kPieceQueue] = make_uint4(bar, par, bytes, chunk);
    ++f.tail;
    f.bytes += bytes;
}

// Lane 0 of the producer warpgroup streams every chunk of every task of this
// SM's queue into the ring, one task record ahead.
__device__ void producer_loop(const KParams &p, const SmemLayout &s, int qb, int qe)
{
    const uint64_t pol_w = evict_first_policy();  // weights: streamed once per step
    const int NS = p.ring_stages;
    uint32_t k = 0;  // chunks issued
    int pst = 0;          // stage of chunk k (k % NS)
    uint32_t ppar = 0u;   // phase of chunk k's full barriers ((k / NS) & 1)
    volatile int *abort_flag = s.flags;
    bool stop = false;
    uint64_t prof_wait = 0, prof_bytes = 0, prof_setup = 0;
    uint64_t cpos = 0;  // stream position of the copy cursor
    Lookahead la{};
    la.ti = qb - 1;
    la.part = 2;
    Flight fl{0u, 0u, 0u};
    if (p.ffn_fused && !p.dpack && p.dmaps) {
        // the Wdown tensor maps sit in global memory that the host rewrites
        // before each launch of the no-allocation step: order those writes
        // before this launch's first tensor copies through them
        for (int l = 0; l < p.n_layers; ++l)
            tmap_acquire(static_cast<const uint8_t *>(p.dmaps) + (size_t)l * 128);
    }
    if (qb < qe)
        stage_task(s.ptask_a, p.tasks + qb);
    for (int ti = qb; ti < qe && !stop; ++ti) {
        const uint64_t ts = p.prof ? gtimer() : 0;
        const uint64_t wait_before = prof_wait;
        stage_task_wait();
        const TaskDesc d = read_staged(s.ptask_a + ((ti - qb) & 1) * sizeof(TaskDesc));
        if (ti + 1 < qe)  // the next record streams in while this task's chunks issue
            stage_task(s.ptask_a + ((ti + 1 - qb) & 1) * sizeof(TaskDesc), p.tasks + ti + 1);
        const Geom g = task_geom(p, d);
        const uint8_t *w0 = static_cast<const uint8_t *>(d.w0);
        const uint8_t *w1 = static_cast<const uint8_t *>(d.w1);
        for (int i = 0; i < g.nchunks; ++i, ++k) {
            const int st = pst;
            const uint32_t done_below = k >= (uint32_t)NS ? k - NS + 1 : 0u;
            if (k >= (uint32_t)NS) {
                const uint32_t par = ppar ^ 1u;  // the stage's previous use
                uint32_t it = 0;
                uint64_t t0 = 0;
                while (!mbar_try_wait(s.empty_a + 8 * st, par)) {
                    if (it == 0) {
                        t0 = gtimer();
                        if (p.lookahead)
                            lookahead_pump(p, la, qe, cpos, cpos + p.lookahead);
                    }
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
                if (p.prof && it)
                    prof_wait += gtimer() - t0;
            }
            const uint32_t dst = s.ring_a + (uint32_t)st * p.stage_bytes;
            const uint32_t bar0 = s.full_a + 8 * (st * kPieces);
            const uint32_t par = ppar;
            if (++pst == NS) {  // the stage and phase of the next chunk
                pst = 0;
                ppar ^= 1u;
            }
            if (p.prof && i == 0)  // time from the task's start to its first copy
                prof_setup += (gtimer() - ts) - (prof_wait - wait_before);
            int used = 0;  // piece barriers armed for this chunk
            if (d.kind == TK_ATTN) {
                // K rows on piece 0, V rows on piece 1
                const int a = g.pa + i * g.P;
                const int b = min(a + g.P, g.pb);
                const uint32_t nb = (uint32_t)(b - a) * p.head_dim * 2;
                for (int h = 0; h < 2 && !stop; ++h) {
                    if (!flight_reserve(p, s, fl, nb, done_below, prof_wait)) {
                        stop = true;
                        break;
                    }
                    const uint32_t bar = bar0 + 8 * h;
                    mbar_arrive_expect_tx(bar, nb);
                    bulk_g2s_nohint(dst + (uint32_t)h * g.P * p.head_dim * 2,
                                    (h ? w1 : w0) + (size_t)a * p.head_dim * 2, nb, bar);
                    flight_push(s, fl, bar, par, nb, k);
                    ++used;
                }
                prof_bytes += 2 * nb;
                cpos += 2 * nb;
            } else if (i >= g.ngu) {
                // fused FFN, Wdown part: rows [r0w, r0w + nrows) of the slice's
                // 16-byte column groups jb, at (jb nrows + row) * 16 in the stage:
                // one bulk copy per group from the packed copy, or TMA boxes of
                // 16 bytes x br rows from the caller's Wdown; all on piece 0
                const int r0w = (i - g.ngu) * g.rpc2;
                const int nrows = min(g.rpc2, p.hidden - r0w);
                const uint32_t nb = (uint32_t)(nrows * g.ncb * 16);
                if (!flight_reserve(p, s, fl, nb, done_below, prof_wait)) {
                    stop = true;
                } else {
                    mbar_arrive_expect_tx(bar0, nb);
                    if (p.dpack) {
                        const uint8_t *src = p.dpack +
                                             (size_t)d.layer * p.hidden * p.ffn * g.esz +
                                             ((size_t)(d.r0 / (16 / g.esz)) * p.hidden + r0w) * 16;
                        for (int jb = 0; jb < g.ncb; ++jb)
                            bulk_g2s(dst + (uint32_t)(jb * nrows * 16),
                                     src + (size_t)jb * p.hidden * 16, (uint32_t)nrows * 16,
                                     bar0, pol_w);
                    } else {
                        const int br = p.ffn_box_rows;
                        const void *tmap =
                            static_cast<const uint8_t *>(p.dmaps) + (size_t)d.layer * 128;
                        for (int ib = 0; ib < nrows / br; ++ib)
                            for (int jb = 0; jb < g.ncb; ++jb)
                                tma_load_2d(dst + (uint32_t)((jb * nrows + ib * br) * 16), tmap,
                                            d.r0 + jb * (16 / g.esz), r0w + ib * br, bar0,
                                            pol_w);
                    }
                    flight_push(s, fl, bar0, par, nb, k);
                    used = 1;
                }
                prof_bytes += nb;
                cpos += nb;
            } else {
                // GEMV rows: one contiguous range, split into up to kPieces
                // pieces of about p.piece bytes (multiples of 16 bytes)
                const int part = i / g.nck, c = i % g.nck;
                const int r = c * g.rpc;
                const int nr = min(g.rpc, g.R - r);
                const uint32_t nb = (uint32_t)nr * g.RB;
                const uint8_t *src = (part ? w1 : w0) + (size_t)r * g.RB;
                const uint32_t np = max(1u, min((uint32_t)kPieces, (nb + p.piece - 1) / p.piece));
                const uint32_t ps = ((nb + np - 1) / np + 15u) & ~15u;
                for (uint32_t pc = 0; pc < np; ++pc) {
                    const uint32_t off = pc * ps;
                    if (off >= nb)
                        break;
                    const uint32_t len = min(ps, nb - off);
                    if (!flight_reserve(p, s, fl, len, done_below, prof_wait)) {
                        stop = true;
                        break;
                    }
                    const uint32_t bar = bar0 + 8 * pc;
                    mbar_arrive_expect_tx(bar, len);
                    bulk_g2s(dst + off, src + off, len, bar, pol_w);
                    flight_push(s, fl, bar, par, len, k);
                    ++used;
                }
                prof_bytes += nb;
                cpos += nb;
            }
            // the chunk's unused piece barriers complete this phase at once (on
            // an abort too, so that the drain below can wait for the chunk)
            for (int pc = used; pc < kPieces; ++pc)
                mbar_arrive(bar0 + 8 * pc);
            if (stop) {
                ++k;
                break;
            }
        }
    }
    if (p.prof) {
        unsigned long long *pc = p.prof + (size_t)blockIdx.x * kProfKinds * kProfFields;
        pc[2] = prof_wait;
        pc[3] = gtimer();
        pc[4] = prof_bytes;
        pc[5] = prof_setup;
    }
    // Drain: wait (bounded) for the copies still in flight so that no bulk
    // copy writes into shared memory after this CTA has exited.
    const uint32_t first = k > (uint32_t)NS ? k - NS : 0;
    for (uint32_t j = first; j < k; ++j) {
        const int st = j % NS;
        const uint32_t par = (j / NS) & 1;
        for (int pc = 0; pc < kPieces; ++pc) {
            uint32_t it = 0;
            const uint64_t t1 = gtimer();
            while (!mbar_try_wait(s.full_a + 8 * (st * kPieces + pc), par)) {
                if ((++it & 255) == 0 && (gtimer() - t1 > p.timeout_ns || it > (1u << 30)))
                    break;
            }
        }
    }
}

// ------------------------------------------------------------------ consumers
// The consumers' position in the ring: chunk k sits in stage st = k % stages,
// whose full barrier completes phase par = (k / stages) & 1 for it.  Advanced
// one chunk at a time, so that no chunk pays for a division by the run-time
// stage count.
struct RingPos {
    uint32_t k;
    int st;
    uint32_t par;
    __device__ __forceinline__ void advance(int stages)
    {
        ++k;
        if (++st == stages) {
            st = 0;
            par ^= 1u;
        }
    }
};

// Waits (all lanes of a warp together) until the ring stage of chunk kc is
// full: lane l polls piece l % kPieces of the stage, so one SIMT poll covers
// every piece barrier.
__device__ __forceinline__ bool wait_full(const KParams &p, const SmemLayout &s, const RingPos &kc)
{
    const int st = kc.st;
    const uint32_t par = kc.par;
    const uint32_t bar = s.full_a + 8 * (st * kPieces + (threadIdx.x & (kPieces - 1)));
    volatile int *abort_flag = s.flags;
    uint32_t it = 0;
    uint64_t t0 = 0;
    while (true) {
        const bool ok = mbar_try_wait(bar, par);
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
                                              const RingPos &kc, int lane)
{
    __syncwarp();
    if (lane == 0)
        mbar_arrive(s.empty_a + 8 * kc.st);
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

// A flagged read gives up on an abort of this CTA, on an error another SM
// recorded, or after the wait limit, which it records (code 1, no counter;
// seen = the tag it last found, target = this step's).  s.flags[2] holds the
// index of the CTA's current task.
__device__ __forceinline__ void fw_record_timeout(const KParams &p, const SmemLayout &s,
                                               uint64_t last)
{
    record_error(p, 1u, *reinterpret_cast<volatile int *>(s.flags + 2), -1,
                 (uint32_t)(last >> 32), p.tag);
}
__device__ __forceinline__ bool fw_give_up(const KParams &p, const SmemLayout &s, uint64_t t0,
                                           uint64_t last, uint32_t it)
{
    if (*reinterpret_cast<volatile int *>(s.flags) != 0 || ld_relaxed(&p.err->code) != 0u)
        return true;
    if (gtimer() - t0 > p.timeout_ns || it > (1u << 26)) {
        fw_record_timeout(p, s, last);
        return true;
    }
    return false;
}

// Phase timers: consumer thread 0 adds the time it spent polling flagged
// words past the first load (the task's wait for its inputs) to a 64-bit
// slot at s.flags + 4, which the consumer loop clears at each task.
__device__ __forceinline__ void fw_note(const KParams &p, const SmemLayout &s, uint64_t t0)
{
    if (p.prof && threadIdx.x == kProducerThreads) {
        volatile unsigned long long *a =
            reinterpret_cast<volatile unsigned long long *>(s.flags + 4);
        *a = *a + (gtimer() - t0);
    }
}

// Thread ct's elements i = ct + 256 j (j < NJ, i < n) of a flagged vector:
// all loads go out at once, then the words still without this step's tag are
// loaded again, all at once, until every one has it.  False when the read
// gave up (the caller raises the CTA's abort flag before its next barrier).
template <int NJ>
__device__ __forceinline__ bool fw_read_strided(const KParams &p, const SmemLayout &s,
                                                const uint64_t *src, int n, int ct,
                                                float (&xv)[NJ])
{
    static_assert(NJ <= 32, "pending bits");
    const uint32_t tag = p.tag;
    uint64_t w[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        const int i = ct + j * kConsumerThreads;
        w[j] = i < n ? fw_ld(src + i) : (uint64_t)tag << 32;
    }
    uint32_t pend = 0u;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        xv[j] = fw_val(w[j]);
        if (!fw_ok(w[j], tag))
            pend |= 1u << j;
    }
    uint64_t t0 = 0;
    // (the words are usually there by the first load once the task's inputs
    // are complete; the compiler is told so, to keep this loop out of the
    // straight-line code)
    for (uint32_t it = 0; __builtin_expect(pend != 0u, 0); ++it) {
        if (it == 0)
            t0 = gtimer();
#pragma unroll
        for (int j = 0; j < NJ; ++j)
            if (pend & (1u << j))
                w[j] = fw_ld(src + ct + j * kConsumerThreads);
        uint64_t last = 0;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            if (pend & (1u << j)) {
                if (fw_ok(w[j], tag)) {
                    xv[j] = fw_val(w[j]);
                    pend &= ~(1u << j);
                } else {
                    last = w[j];
                }
            }
        }
        if (pend && (it & 15) == 15 && fw_give_up(p, s, t0, last, it))
            return false;
    }
    if (t0)
        fw_note(p, s, t0);
    return true;
}

// The words at a[j] (null: none, value 0) of flagged vectors, as above.
template <int N>
__device__ __forceinline__ bool fw_gather(const KParams &p, const SmemLayout &s,
                                          const uint64_t *const (&a)[N], float (&v)[N])
{
    const uint32_t tag = p.tag;
    uint64_t w[N];
#pragma unroll
    for (int j = 0; j < N; ++j)
        w[j] = a[j] ? fw_ld(a[j]) : (uint64_t)tag << 32;
    uint32_t pend = 0u;
#pragma unroll
    for (int j = 0; j < N; ++j) {
        v[j] = fw_val(w[j]);
        if (!fw_ok(w[j], tag))
            pend |= 1u << j;
    }
    uint64_t t0 = 0;
    // (the words are usually there by the first load once the task's inputs
    // are complete; the compiler is told so, to keep this loop out of the
    // straight-line code)
    for (uint32_t it = 0; __builtin_expect(pend != 0u, 0); ++it) {
        if (it == 0)
            t0 = gtimer();
#pragma unroll
        for (int j = 0; j < N; ++j)
            if (pend & (1u << j))
                w[j] = fw_ld(a[j]);
        uint64_t last = 0;
#pragma unroll
        for (int j = 0; j < N; ++j) {
            if (pend & (1u << j)) {
                if (fw_ok(w[j], tag)) {
                    v[j] = fw_val(w[j]);
                    pend &= ~(1u << j);
                } else {
                    last = w[j];
                }
            }
        }
        if (pend && (it & 15) == 15 && fw_give_up(p, s, t0, last, it))
            return false;
    }
    if (t0)
        fw_note(p, s, t0);
    return true;
}

// A GEMV lane's activations from the 32-bit flagged SwiGLU words: vector
// v = vb + lane + 32 i (i < ni; zeros for the others) holds the E elements at
// xg + v E, read G = min(E, 4) words at a time, in rounds of RI vectors (a
// bf16 or int8 lane with more than 48 activations takes two, to bound the
// registers a round holds; an int4 lane's 64 take one);
// every load of a round goes out before any word of it is looked at, and
// groups still without this step's tag are loaded again until all have it.
template <int NI, int E, int RI>
__device__ __forceinline__ bool fw_lane_round(const KParams &p, const SmemLayout &s,
                                              const uint32_t *xg, int vb, int ni, int lane,
                                              int i0, float (&xf)[NI][E])
{
    constexpr int G = E < 4 ? E : 4;
    constexpr int H = E / G;  // groups per vector
    static_assert(E % G == 0 && (G == 2 || G == 4) && RI * H <= 32, "pending bits");
    const uint32_t t8 = fw8_tag(p.tag);
    uint32_t w[RI][H][G];
#pragma unroll
    for (int r = 0; r < RI; ++r) {
        const uint32_t *vp = xg + (size_t)(vb + lane + 32 * (i0 + r)) * E;
#pragma unroll
        for (int h = 0; h < H; ++h) {
#pragma unroll
            for (int q = 0; q < G; ++q)
                w[r][h][q] = t8;  // a zero with this step's tag
            if (i0 + r < ni) {
                if constexpr (G == 4)
                    fw32_ld4(vp + 4 * h, w[r][h]);
                else
                    fw32_ld2(vp + 2 * h, w[r][h]);
            }
        }
    }
    uint32_t pend = 0u;
#pragma unroll
    for (int r = 0; r < RI; ++r)
#pragma unroll
        for (int h = 0; h < H; ++h) {
            bool ok = true;
#pragma unroll
            for (int q = 0; q < G; ++q) {
                xf[i0 + r][G * h + q] = fw32_val(w[r][h][q]);
                ok = ok && fw32_ok(w[r][h][q], t8);
            }
            if (!ok)
                pend |= 1u << (r * H + h);
        }
    uint64_t t0 = 0;
    for (uint32_t it = 0; __builtin_expect(pend != 0u, 0); ++it) {
        if (it == 0)
            t0 = gtimer();
#pragma unroll
        for (int r = 0; r < RI; ++r) {
            const uint32_t *vp = xg + (size_t)(vb + lane + 32 * (i0 + r)) * E;
#pragma unroll
            for (int h = 0; h < H; ++h)
                if (pend & (1u << (r * H + h))) {
                    if constexpr (G == 4)
                        fw32_ld4(vp + 4 * h, w[r][h]);
                    else
                        fw32_ld2(vp + 2 * h, w[r][h]);
                }
        }
        uint32_t last = 0;
#pragma unroll
        for (int r = 0; r < RI; ++r)
#pragma unroll
            for (int h = 0; h < H; ++h) {
                const uint32_t bit = 1u << (r * H + h);
                if (pend & bit) {
                    bool ok = true;
#pragma unroll
                    for (int q = 0; q < G; ++q)
                        ok = ok && fw32_ok(w[r][h][q], t8);
                    if (ok) {
#pragma unroll
                        for (int q = 0; q < G; ++q)
                            xf[i0 + r][G * h + q] = fw32_val(w[r][h][q]);
                        pend &= ~bit;
                    } else {
                        last = w[r][h][0];
                    }
                }
            }
        if (pend && (it & 15) == 15 &&
            fw_give_up(p, s, t0, (uint64_t)(last & 0xffu) << 32, it))
            return false;
    }
    if (t0)
        fw_note(p, s, t0);
    return true;
}

template <int NI, int E>
__device__ __forceinline__ bool fw_lane_vectors(const KParams &p, const SmemLayout &s,
                                                const uint32_t *xg, int vb, int ni, int lane,
                                                float (&xf)[NI][E])
{
    constexpr int RI = NI * E > 48 && E < 32 && NI > 1 ? (NI + 1) / 2 : NI;
    if (!fw_lane_round<NI, E, RI>(p, s, xg, vb, ni, lane, 0, xf))
        return false;
    if constexpr (RI < NI)
        return fw_lane_round<NI, E, NI - RI>(p, s, xg, vb, ni, lane, RI, xf);
    return true;
}

// Counter wait by consumer thread 0; returns false on timeout / abort.
__device__ bool wait_counter(const KParams &p, const TaskDesc &d, int ti)
{
    if (d.wait_ctr < 0)
        return true;
    const uint32_t target = p.epoch * d.wait_total + d.wait_count;
    const uint32_t *ctr = p.counters + d.wait_ctr;
    uint64_t t0 = 0;
    uint32_t v = 0;
    for (uint32_t it = 0;; ++it) {
        v = ld_acquire(ctr);
        if ((int32_t)(v - target) >= 0)
            return true;
        if (it == 0)
            t0 = gtimer();
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

// Block-wide sum over the 256 consumer threads, through s.scr[16 .. 24),
// which nothing else uses: one barrier (the next call comes after the
// caller's own barriers, so the slots are free again by then).
__device__ float block_sum(float v, const SmemLayout &s, int ct)
{
    v = warp_sum(v);
    if ((ct & 31) == 0)
        s.scr[16 + (ct >> 5)] = v;
    consumer_bar();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w)
        t += s.scr[16 + w];
    return t;
}

// vec[i] = g_i * x_i / sqrt(mean x^2 + eps), x from flagged words, the
// fixed-point residual or the embedding row (bf16).  The gains gv (thread t:
// elements t + 256 j, raw bf16 bits, first used here) were loaded before the
// task's wait, so that their first touch in HBM is off the critical path;
// every load of x is issued before
// any store (one L2 round trip once the words are there); hidden <=
// kMaxPerThread * 256.
constexpr int kMaxPerThread = 16;
__device__ void rmsnorm_prologue(const KParams &p, const SmemLayout &s, const uint64_t *x_fw,
                                 const uint16_t *x_bf16, const long long *x_fix,
                                 const uint32_t (&gv)[kMaxPerThread], int ct)
{
    const int n = p.hidden;
    float xv[kMaxPerThread];
    if (x_fw) {
        if (!fw_read_strided<kMaxPerThread>(p, s, x_fw, n, ct, xv))
            s.flags[0] = 1;  // before block_sum's barrier: every thread sees it after
    } else {
#pragma unroll
        for (int j = 0; j < kMaxPerThread; ++j) {
            const int i = ct + j * kConsumerThreads;
            xv[j] = 0.f;
            if (i < n)
                xv[j] = x_fix ? from_fix(__ldcg(x_fix + i)) : bf16_to_f(__ldg(x_bf16 + i));
        }
    }
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxPerThread; ++j)
        ss = fmaf(xv[j], xv[j], ss);
    const float tot = block_sum(ss, s, ct);
    const float inv = rsqrtf(tot / (float)n + p.rms_eps);
#pragma unroll
    for (int j = 0; j < kMaxPerThread; ++j) {
        const int i = ct + j * kConsumerThreads;
        if (i < n)
            s.vec[vidx(i)] = bf16_to_f((uint16_t)gv[j]) * (xv[j] * inv);
    }
    consumer_bar();
}

// GEMV over a task's chunks.  Warp w = rg + RG * ks owns K-slice ks (vectors
// [vb, ve) of every row, lane l holding vb + l + 32 i with its activations in
// registers as float pairs) of the rows j = rg, rg + RG, ... of each chunk,
// two rows at a time, and writes the slice's row sum to red[w][row]; the
// epilogue adds the KS slices of a row.  The activations come from the
// shared vector (prologue output) or, when xg is set, straight from L2.
template <int ESZ, int VB>
__device__ __forceinline__ bool gemv_task(const KParams &p, const SmemLayout &s, const Geom g,
                                          RingPos &kc, int warp, int lane, const uint32_t *xg,
                                          uint64_t *wt)
{
    constexpr int E = VB / ESZ;   // elements per vector (even)
    constexpr int NI = 64 / E;    // vectors per lane at most (64 activations)
    constexpr int EP = E / 2;     // float pairs per vector
    const int NV = g.RB / VB;
    const int VPS = (NV + g.KS - 1) / g.KS;
    const int RG = g.RG, RB = g.RB, rpc = g.rpc, R = g.R, nck = g.nck;
    const int rg = warp % RG, ks = warp / RG;
    const int vb = ks * VPS;
    const int ve = min(vb + VPS, NV);
    const int ni = (ve - vb - lane + 31) / 32;  // vectors this lane holds (may be <= 0)
    // the lane's activations: 16-byte pieces of its vectors (8 bytes when a
    // vector holds 2 elements), from the padded shared vector or from the
    // flagged words xg
    f2_t xp[NI][EP];
    if (xg) {
        float xf[NI][E];
        if (!fw_lane_vectors<NI, E>(p, s, xg, vb, ni, lane, xf))
            return false;
#pragma unroll
        for (int i = 0; i < NI; ++i)
#pragma unroll
            for (int e = 0; e < EP; ++e)
                xp[i][e] = pk2(xf[i][2 * e], xf[i][2 * e + 1]);
    } else {
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            const int v = vb + lane + 32 * i;
            if constexpr (E >= 4) {
#pragma unroll
                for (int e = 0; e < E; e += 4) {
                    float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (i < ni) {
                        const uint4 u = lds128(s.vec_a + (uint32_t)vidx(v * E + e) * 4);
                        t = make_float4(__uint_as_float(u.x), __uint_as_float(u.y),
                                        __uint_as_float(u.z), __uint_as_float(u.w));
                    }
                    xp[i][e / 2] = pk2(t.x, t.y);
                    xp[i][e / 2 + 1] = pk2(t.z, t.w);
                }
            } else {
                float a = 0.f, b = 0.f;
                if (i < ni) {
                    const uint2 t = lds64(s.vec_a + (uint32_t)vidx(v * E) * 4);
                    a = __uint_as_float(t.x);
                    b = __uint_as_float(t.y);
                }
                xp[i][0] = pk2(a, b);
            }
        }
    }
    const uint32_t red_a = s.red_a + (uint32_t)warp * kMaxTaskRows * 4;
    const int SB = p.stage_bytes;
    uint64_t tA = 0, tB = 0;
    for (int i = 0; i < g.ngu; ++i) {
        if (wt)
            tA = gtimer();
        if (!wait_full(p, s, kc))
            return false;
        if (wt) {
            tB = gtimer();
            wt[0] += tB - tA;
        }
        const uint32_t stage_a = s.ring_a + (uint32_t)kc.st * SB;
        const int part = i / nck, c = i - part * nck;
        const int r = c * rpc;
        const int nr = min(rpc, R - r);
        const int rowbase = part * R + r;
        const uint32_t lane_a = stage_a + (uint32_t)(vb + lane) * VB;
        // bf16 interleaves two rows per warp (two reduction chains); int8
        // needs the registers for unpacking and takes one row at a time
        constexpr int ROWS = (ESZ == 2) ? 2 : 1;
        for (int j = rg; j < nr; j += ROWS * RG) {
            const bool two = ROWS == 2 && j + RG < nr;
            const uint32_t ra = lane_a + (uint32_t)j * RB;
            const uint32_t rb = ra + (uint32_t)RG * RB;
            f2_t acc_a[4] = {0ull, 0ull, 0ull, 0ull}, acc_b[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int t0 = 0; t0 < NI; t0 += 4) {
                WVec<VB> wa[4], wb[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (t0 + u < NI && t0 + u < ni) {
                        wa[u] = ldw<VB>(ra + (uint32_t)(t0 + u) * 32 * VB);
                        if (two)
                            wb[u] = ldw<VB>(rb + (uint32_t)(t0 + u) * 32 * VB);
                    }
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (t0 + u < NI && t0 + u < ni) {
                        acc_a[u] = vdot2<ESZ, VB>(wa[u], xp[t0 + u], acc_a[u]);
                        if (two)
                            acc_b[u] = vdot2<ESZ, VB>(wb[u], xp[t0 + u], acc_b[u]);
                    }
            }
            float sa = (sum2(acc_a[0]) + sum2(acc_a[1])) + (sum2(acc_a[2]) + sum2(acc_a[3]));
            float sb = (sum2(acc_b[0]) + sum2(acc_b[1])) + (sum2(acc_b[2]) + sum2(acc_b[3]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                sa += __shfl_xor_sync(0xffffffffu, sa, o);
                sb += __shfl_xor_sync(0xffffffffu, sb, o);
            }
            if (lane == 0) {
                stsf(red_a + (uint32_t)(rowbase + j) * 4, sa);
                if (two)
                    stsf(red_a + (uint32_t)(rowbase + j + RG) * 4, sb);
            }
        }
        release_stage(p, s, kc, lane);
        kc.advance(p.ring_stages);
        if (wt)
            wt[1] += gtimer() - tB;
    }
    return true;
}

// Sums RW per-lane row partials over the warp with a transposed exchange:
// the first log2(RW) steps trade halves of the rows between lane groups, so
// four rows cost six shuffles and two rows five, instead of five per row.
// Afterwards every lane of group l >> (5 - log2 RW) holds that row's total.
template <int RW>
__device__ __forceinline__ float warp_rows_sum(float (&s)[RW], int lane)
{
    constexpr unsigned FULL = 0xffffffffu;
    if constexpr (RW == 4) {
        const bool up = lane & 16;
        s[0] = (up ? s[2] : s[0]) + __shfl_xor_sync(FULL, up ? s[0] : s[2], 16);
        s[1] = (up ? s[3] : s[1]) + __shfl_xor_sync(FULL, up ? s[1] : s[3], 16);
        const bool up8 = lane & 8;
        s[0] = (up8 ? s[1] : s[0]) + __shfl_xor_sync(FULL, up8 ? s[0] : s[1], 8);
#pragma unroll
        for (int o = 4; o > 0; o >>= 1)
            s[0] += __shfl_xor_sync(FULL, s[0], o);
    } else if constexpr (RW == 2) {
        const bool up = lane & 16;
        s[0] = (up ? s[1] : s[0]) + __shfl_xor_sync(FULL, up ? s[0] : s[1], 16);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1)
            s[0] += __shfl_xor_sync(FULL, s[0], o);
    } else {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            s[0] += __shfl_xor_sync(FULL, s[0], o);
    }
    return s[0];
}

// int16 x int8 two-way dot products into an int32 accumulator: the 16-bit
// halves of a times bytes 0, 1 (lo) or 2, 3 (hi) of b.
__device__ __forceinline__ int dp2a_lo(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp2a.lo.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ int dp2a_hi(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp2a.hi.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// The lane's activations for a GEMV with 16-byte weight vectors.  bf16
// weights: f[i][e], element e of vector i as a float.  int8 weights: the
// lane quantises its own activations to int16 with one scale (|error| <= half
// a step = max|x| / 65534 per element) and packs them in pairs, q[i][k] =
// elements 2k, 2k + 1 of vector i; the int8 x int16 products then add up
// exactly in int32 (a lane's sum stays below 64 * 127 * 32767 < 2^31).
//
// Packed int4 weights (ESZ = 0): 32 codes per vector.  The activations are
// quantised the same way and packed in the order the nibble split of
// gemv_rows needs: for the 8 elements 8k .. 8k + 7 of a vector, q[i][4k ..
// 4k + 3] = (0, 2), (4, 6), (1, 3), (5, 7); xs[i] = 8 x the sum of the
// vector's int16 activations (the bias the offset codes carry).
template <int ESZ, int NI_>
struct LaneX {
    static constexpr int E = ESZ ? 16 / ESZ : 32;  // elements per vector
    static constexpr int NI = NI_;       // vectors per lane at most (NI E <= 64 activations)
    float f[ESZ == 2 ? NI : 1][ESZ == 2 ? E : 1];
    uint32_t q[ESZ == 2 ? 1 : NI][ESZ == 0 ? 16 : 8];
    int xs[ESZ == 0 ? NI : 1];
    float scale;                         // int8 / int4: value of one int16 step
};

// int16 pairs of a times unsigned bytes 0, 1 (lo) or 2, 3 (hi) of b.
__device__ __forceinline__ int dp2a_lo_u(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ int dp2a_hi_u(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ uint32_t pack_i16(int a, int b)
{
    return ((uint32_t)a & 0xffffu) | ((uint32_t)b << 16);
}

// Rows j0 + RG r (r < RW) of a ring chunk against the lane's activations;
// each row's warp total goes to red[rowbase + row] (the warp's red slice).
// The lane reads vector i of a row at byte voff[i] of it: every lane takes
// all NI vectors, with no guard in the loop (a lane's vectors past the end of
// its K-slice re-read a vector of the slice and meet zero activations), so
// that the compiler can issue the loads of all RW rows ahead of the math.
template <int ESZ, int NI, int RW>
__device__ __forceinline__ void gemv_rows(const LaneX<ESZ, NI> &x, uint32_t stage_a,
                                          const uint32_t (&voff)[NI], const uint32_t (&soff)[NI],
                                          int RB, int RG, int j0, uint32_t red_a, int rowbase,
                                          int lane)
{
    float sr[RW];
    uint32_t ra[RW];
#pragma unroll
    for (int r = 0; r < RW; ++r)
        ra[r] = stage_a + (uint32_t)((j0 + r * RG) * RB);
    if constexpr (ESZ == 0) {
        // int4: XOR 0x8 per nibble turns 4-bit two's complement into code + 8;
        // even and odd codes as unsigned bytes, dp2a against the int16 pairs,
        // minus the bias, exact in int32 (|sum| < 32 * 15 * 32767); then the
        // vector's group scale (at byte soff[i] of the row) in fp32
        float acc[RW][2];
#pragma unroll
        for (int r = 0; r < RW; ++r)
            acc[r][0] = acc[r][1] = 0.f;
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            uint4 w[RW];
            float sc[RW];
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                w[r] = lds128(ra[r] + voff[i]);
                sc[r] = fp16_to_f((uint16_t)lds16(ra[r] + soff[i]));
            }
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                const uint32_t A[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
                int s0 = 0, s1 = 0;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t t = A[q] ^ 0x88888888u;
                    const uint32_t lo = t & 0x0f0f0f0fu;
                    const uint32_t hi = (t >> 4) & 0x0f0f0f0fu;
                    s0 = dp2a_lo_u(x.q[i][4 * q], lo, s0);
                    s1 = dp2a_hi_u(x.q[i][4 * q + 1], lo, s1);
                    s0 = dp2a_lo_u(x.q[i][4 * q + 2], hi, s0);
                    s1 = dp2a_hi_u(x.q[i][4 * q + 3], hi, s1);
                }
                acc[r][i & 1] = fmaf((float)(s0 + s1 - x.xs[i]), sc[r], acc[r][i & 1]);
            }
        }
#pragma unroll
        for (int r = 0; r < RW; ++r)
            sr[r] = (acc[r][0] + acc[r][1]) * x.scale;
    } else if constexpr (ESZ == 2) {
        float acc[RW][4];
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int q = 0; q < 4; ++q)
                acc[r][q] = 0.f;
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            uint4 w[RW];
#pragma unroll
            for (int r = 0; r < RW; ++r)
                w[r] = lds128(ra[r] + voff[i]);
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                const uint32_t A[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc[r][q] = fmaf(__uint_as_float(A[q] << 16), x.f[i][2 * q], acc[r][q]);
                    acc[r][q] = fmaf(__uint_as_float(A[q] & 0xffff0000u), x.f[i][2 * q + 1],
                                     acc[r][q]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < RW; ++r)
            sr[r] = (acc[r][0] + acc[r][1]) + (acc[r][2] + acc[r][3]);
    } else {
        int acc[RW][2];
#pragma unroll
        for (int r = 0; r < RW; ++r)
            acc[r][0] = acc[r][1] = 0;
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            uint4 w[RW];
#pragma unroll
            for (int r = 0; r < RW; ++r)
                w[r] = lds128(ra[r] + voff[i]);
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                const uint32_t A[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc[r][0] = dp2a_lo(x.q[i][2 * q], A[q], acc[r][0]);
                    acc[r][1] = dp2a_hi(x.q[i][2 * q + 1], A[q], acc[r][1]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < RW; ++r)
            sr[r] = (float)(acc[r][0] + acc[r][1]) * x.scale;
    }
    const float tot = warp_rows_sum<RW>(sr, lane);
    constexpr int SH = RW == 4 ? 3 : RW == 2 ? 4 : 5;
    if ((lane & ((1 << SH) - 1)) == 0)
        stsf(red_a + (uint32_t)(rowbase + j0 + (lane >> SH) * RG) * 4, tot);
}

// GEMV over a task's chunks with 16-byte weight vectors (every shape whose
// rows are a multiple of 16 bytes).  Warp w = rg + RG ks owns K-slice ks of
// the rows rg, rg + RG, ... of every chunk, and takes them four at a time
// (then two, then one): four independent rows per weight-vector load and
// four accumulators per row keep the FMA or dp2a pipes fed, and one
// transposed shuffle reduction serves the four rows.  NI (vectors a lane
// holds) is a template parameter so that the activation registers are sized
// to the shape, not to the largest one.
template <int ESZ, int NI>
__device__ __forceinline__ bool gemv16_task(const KParams &p, const SmemLayout &s, const Geom g,
                                            RingPos &kc, int warp, int lane, const uint32_t *xg,
                                            uint64_t *wt)
{
    using LX = LaneX<ESZ, NI>;
    constexpr int E = LX::E;
    const int NV = ESZ ? g.RB >> 4 : g.K >> 5;  // int4 rows: code vectors, then the scales
    const int VPS = (NV + g.KS - 1) >> g.ks_log2;
    const int RG = g.RG, RB = g.RB, rpc = g.rpc, R = g.R, nck = g.nck;
    const int rg = warp & (RG - 1), ks = warp >> g.rg_log2;
    const int vb = ks * VPS;
    const int ve = min(vb + VPS, NV);
    const int ni = (ve - vb - lane + 31) >> 5;  // vectors this lane holds (may be <= 0)
    LX x;
    {
        float xf[NI][E];
        if (xg) {
            if (!fw_lane_vectors<NI, E>(p, s, xg, vb, ni, lane, xf))
                return false;
        } else {
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                const int v = vb + lane + 32 * i;
#pragma unroll
                for (int e = 0; e < E; e += 4) {
                    uint4 u = make_uint4(0u, 0u, 0u, 0u);
                    if (i < ni)
                        u = lds128(s.vec_a + (uint32_t)vidx(v * E + e) * 4);
                    xf[i][e] = __uint_as_float(u.x);
                    xf[i][e + 1] = __uint_as_float(u.y);
                    xf[i][e + 2] = __uint_as_float(u.z);
                    xf[i][e + 3] = __uint_as_float(u.w);
                }
            }
        }
        if constexpr (ESZ == 2) {
#pragma unroll
            for (int i = 0; i < NI; ++i)
#pragma unroll
                for (int e = 0; e < E; ++e)
                    x.f[i][e] = xf[i][e];
            x.scale = 1.f;
        } else if constexpr (ESZ == 0) {
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < NI; ++i)
#pragma unroll
                for (int e = 0; e < E; ++e)
                    amax = fmaxf(amax, fabsf(xf[i][e]));
            const float inv = amax > 0.f ? 32767.f / amax : 0.f;
            x.scale = amax * (1.f / 32767.f);
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                int sum = 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    int v[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        v[e] = max(-32767, min(32767, __float2int_rn(xf[i][8 * k + e] * inv)));
                        sum += v[e];
                    }
                    x.q[i][4 * k] = pack_i16(v[0], v[2]);
                    x.q[i][4 * k + 1] = pack_i16(v[4], v[6]);
                    x.q[i][4 * k + 2] = pack_i16(v[1], v[3]);
                    x.q[i][4 * k + 3] = pack_i16(v[5], v[7]);
                }
                x.xs[i] = 8 * sum;
            }
        } else {
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < NI; ++i)
#pragma unroll
                for (int e = 0; e < E; ++e)
                    amax = fmaxf(amax, fabsf(xf[i][e]));
            const float inv = amax > 0.f ? 32767.f / amax : 0.f;
            x.scale = amax * (1.f / 32767.f);
#pragma unroll
            for (int i = 0; i < NI; ++i)
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int a = max(-32767, min(32767, __float2int_rn(xf[i][2 * k] * inv)));
                    const int b = max(-32767, min(32767, __float2int_rn(xf[i][2 * k + 1] * inv)));
                    x.q[i][k] = ((uint32_t)a & 0xffffu) | ((uint32_t)b << 16);
                }
        }
    }
    // byte offset in a row of the lane's vector i: its own while i < ni,
    // else (zero activations) one that the slice surely holds
    // (int4 rows: the vector's group scale is at soff[i], after the K / 2
    // code bytes of the row, one fp16 per 128 inputs = 4 vectors)
    uint32_t voff[NI], soff[NI];
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        const int v = i < ni ? vb + lane + 32 * i : ni > 0 ? vb + lane : min(vb, NV - 1);
        voff[i] = (uint32_t)v * 16;
        soff[i] = ESZ ? 0u : (uint32_t)(g.K / 2 + 2 * (v >> 2));
    }
    const uint32_t red_a = s.red_a + (uint32_t)warp * kMaxTaskRows * 4;
    const int SB = p.stage_bytes;
    // rows rg + RG m (m < nrw) of a chunk are this warp's: rpc / RG of a full
    // chunk (rpc is a multiple of RG); the last chunk of a part may hold fewer
    const int nrw_full = rpc >> g.rg_log2;
    uint64_t tA = 0, tB = 0;
    int part = 0, cc = 0;  // chunk c = part * nck + cc, advanced without divisions
    for (int c = 0; c < g.ngu; ++c) {
        if (wt)
            tA = gtimer();
        if (!wait_full(p, s, kc))
            return false;
        if (wt) {
            tB = gtimer();
            wt[0] += tB - tA;
        }
        const uint32_t stage_a = s.ring_a + (uint32_t)kc.st * SB;
        const int r0 = cc * rpc;
        const int nr = min(rpc, R - r0);
        const int rowbase = part * R + r0;
        const int nrw = nr == rpc ? nrw_full : nr > rg ? (nr - rg + RG - 1) >> g.rg_log2 : 0;
        if (++cc == nck) {
            cc = 0;
            ++part;
        }
        int m = 0;
        for (; m + 4 <= nrw; m += 4)
            gemv_rows<ESZ, NI, 4>(x, stage_a, voff, soff, RB, RG, rg + RG * m, red_a, rowbase,
                                  lane);
        if (m + 2 <= nrw) {
            gemv_rows<ESZ, NI, 2>(x, stage_a, voff, soff, RB, RG, rg + RG * m, red_a, rowbase,
                                  lane);
            m += 2;
        }
        if (m < nrw)
            gemv_rows<ESZ, NI, 1>(x, stage_a, voff, soff, RB, RG, rg + RG * m, red_a, rowbase,
                                  lane);
        release_stage(p, s, kc, lane);
        kc.advance(p.ring_stages);
        if (wt)
            wt[1] += gtimer() - tB;
    }
    return true;
}

// Dispatch on the vectors a lane holds for this task's K-slice.
template <int ESZ>
__device__ __forceinline__ bool gemv16(const KParams &p, const SmemLayout &s, const Geom &g,
                                       RingPos &kc, int warp, int lane, const uint32_t *xg,
                                       uint64_t *wt)
{
    const int vps = ((ESZ ? g.RB >> 4 : g.K >> 5) + g.KS - 1) >> g.ks_log2;
    const int nimax = (vps + 31) >> 5;
    if constexpr (ESZ == 0) {
        if (nimax <= 1)
            return gemv16_task<0, 1>(p, s, g, kc, warp, lane, xg, wt);
        return gemv16_task<0, 2>(p, s, g, kc, warp, lane, xg, wt);
    } else if constexpr (ESZ == 2) {
        if (nimax <= 2)
            return gemv16_task<2, 2>(p, s, g, kc, warp, lane, xg, wt);
        if (nimax <= 4)
            return gemv16_task<2, 4>(p, s, g, kc, warp, lane, xg, wt);
        if (nimax <= 6)
            return gemv16_task<2, 6>(p, s, g, kc, warp, lane, xg, wt);
        return gemv16_task<2, 8>(p, s, g, kc, warp, lane, xg, wt);
    } else {
        if (nimax <= 1)
            return gemv16_task<1, 1>(p, s, g, kc, warp, lane, xg, wt);
        if (nimax <= 2)
            return gemv16_task<1, 2>(p, s, g, kc, warp, lane, xg, wt);
        if (nimax <= 3)
            return gemv16_task<1, 3>(p, s, g, kc, warp, lane, xg, wt);
        return gemv16_task<1, 4>(p, s, g, kc, warp, lane, xg, wt);
    }
}

// Fast instances (GENERIC = 0) only run 16-byte weight vectors in the
// model's own format; the generic instance dispatches every variant at run
// time (models with odd row widths, or a bf16 tied head on int8 layers).
template <int Q8, int GENERIC>
__device__ __forceinline__ bool run_gemv(const KParams &p, const SmemLayout &s, const Geom &g,
                                         RingPos &kc, int warp, int lane, const uint32_t *xg,
                                         uint64_t *wt)
{
    if constexpr (!GENERIC) {
        if constexpr (Q8 == 2) {
            if (g.esz == 2)  // a tied LM head stays bf16
                return gemv16<2>(p, s, g, kc, warp, lane, xg, wt);
            return gemv16<0>(p, s, g, kc, warp, lane, xg, wt);
        } else if constexpr (Q8 == 1) {
            return gemv16<1>(p, s, g, kc, warp, lane, xg, wt);
        } else {
            return gemv16<2>(p, s, g, kc, warp, lane, xg, wt);
        }
    } else {
        if (g.esz == 2) {
            if (g.VB == 16)
                return gemv16<2>(p, s, g, kc, warp, lane, xg, wt);
            if (g.VB == 8)
                return gemv_task<2, 8>(p, s, g, kc, warp, lane, xg, wt);
            return gemv_task<2, 4>(p, s, g, kc, warp, lane, xg, wt);
        }
        if (g.VB == 16)
            return gemv16<1>(p, s, g, kc, warp, lane, xg, wt);
        if (g.VB == 8)
            return gemv_task<1, 8>(p, s, g, kc, warp, lane, xg, wt);
        return gemv_task<1, 4>(p, s, g, kc, warp, lane, xg, wt);
    }
}

// Sum of the K-slice partials of output row t (task-relative, parts
// included): the warps rg + RG * ks with rg = (row within its chunk) % RG.
__device__ __forceinline__ float row_total(const SmemLayout &s, const Geom &g, int t)
{
    const int tr = t >= g.R ? t - g.R : t;  // the row within its part (at most two parts)
    const int rg = tr & (g.RG - 1);          // chunks start at multiples of RG
    float y = 0.f;
    for (int ks = 0; ks < g.KS; ++ks)
        y += s.red[(rg + g.RG * ks) * kMaxTaskRows + t];
    return y;
}

// RoPE angle of pair i at position pos (HF rotate_half): a = pos * w_i with
// w_i = theta^(-2i/hd), formed and reduced modulo 2*pi in double precision,
// then sin/cos of the reduced angle in single precision.
__device__ __forceinline__ void rope_angle(int pos, int i, int hd, float theta, float *sn,
                                           float *cs)
{
    const double w = exp2(-(2.0 * i / hd) * log2((double)theta));
    const double a = (double)pos * w;
    const double k = rint(a * 0.15915494309189535);  // a / (2 pi)
    const double r = fma(-k, 6.283185307179586, a);  // a - 2 pi k (|k| small)
    sincosf((float)r, sn, cs);
}

// E consecutive bf16 values at shared address a (2E-byte aligned) as floats.
template <int E>
__device__ __forceinline__ void lds_bf16(uint32_t a, float (&out)[E])
{
    if constexpr (E == 1) {
        out[0] = __uint_as_float(lds16(a) << 16);
    } else if constexpr (E == 2) {
        const uint32_t w = lds32(a);
        out[0] = __uint_as_float(w << 16);
        out[1] = __uint_as_float(w & 0xffff0000u);
    } else if constexpr (E == 4) {
        const uint2 w = lds64(a);
        out[0] = __uint_as_float(w.x << 16);
        out[1] = __uint_as_float(w.x & 0xffff0000u);
        out[2] = __uint_as_float(w.y << 16);
        out[3] = __uint_as_float(w.y & 0xffff0000u);
    } else {
#pragma unroll
        for (int c = 0; c < E / 8; ++c) {
            const uint4 w = lds128(a + c * 16);
            const uint32_t ws_[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                out[c * 8 + 2 * i] = __uint_as_float(ws_[i] << 16);
                out[c * 8 + 2 * i + 1] = __uint_as_float(ws_[i] & 0xffff0000u);
            }
        }
    }
}

// Split-K attention tile for KV head g and chunk c (flash-decoding partial):
// writes (m, l, o[hd]) per query head of the group, unnormalised.
template <int E>
__device__ __forceinline__ bool attn_chunk(const KParams &p, const SmemLayout &s,
                                          const TaskDesc &d, const Geom &g, RingPos &kc,
                                          int ct, int warp, int lane, uint64_t *wt, uint32_t otag)
{
    const int l = d.layer, gi = d.r0, c = d.r1;
    const int hd = p.head_dim, G = p.group, nh = p.n_heads, nkv = p.n_kv_heads;
    const int lph = p.att_lph;  // lanes per head
    float *qs = s.vec;                       // [G][hd], RoPE'd and pre-scaled
    float *kn = qs + G * hd;                 // [hd] new K row (bf16 value)
    float *vn = kn + hd;                     // [hd] new V row (bf16 value)
    float *ws = vn + hd;                     // [8][G][hd + 2] per-warp partials
    const uint64_t *qkv = p.qkv + (size_t)l * p.qkv_rows;
    if (g.j1 <= g.j0)
        return true;  // empty chunk: no partial (the merge skips it)
    // prologue: q of the group's G heads and k get RoPE (pairs i, i + hd/2),
    // q is pre-scaled by 1/sqrt(hd); k and v are rounded to bf16 (the cache
    // format) and chunk 0 appends them at row pos
    const int half = hd / 2;
    const float qscale = rsqrtf((float)hd);
    uint16_t *kd = const_cast<uint16_t *>(static_cast<const uint16_t *>(d.w0)) +
                   (size_t)p.pos * hd;
    uint16_t *vd = const_cast<uint16_t *>(static_cast<const uint16_t *>(d.w1)) +
                   (size_t)p.pos * hd;
    // the flagged words of q, k (as RoPE pairs) and v, two pairs and two v
    // elements per thread and round, all of a round's words polled at once
    // (one round for every head size and group up to (G + 1) hd / 2 <= 512)
    const int npair = (G + 1) * half;
    const uint64_t *vsrc = qkv + (size_t)(nh + nkv) * hd + (size_t)gi * hd;
    for (int r0 = 0; r0 < npair || r0 < hd; r0 += 2 * kConsumerThreads) {
        const uint64_t *a[6];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int i = r0 + ct + k * kConsumerThreads;
            a[2 * k] = a[2 * k + 1] = nullptr;
            if (i < npair) {
                const int hh = i / half, e = i % half;
                const uint64_t *src = hh < G ? qkv + (size_t)(gi * G + hh) * hd
                                             : qkv + (size_t)nh * hd + (size_t)gi * hd;
                a[2 * k] = src + e;
                a[2 * k + 1] = src + e + half;
            }
            a[4 + k] = i < hd ? vsrc + i : nullptr;
        }
        float xv[6];
        if (!fw_gather<6>(p, s, a, xv)) {
            s.flags[0] = 1;
            break;
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int i = r0 + ct + k * kConsumerThreads;
            if (i < npair) {
                const int hh = i / half, e = i % half;
                const float x0 = xv[2 * k], x1 = xv[2 * k + 1];
                float sn, cs;
                rope_angle(p.pos, e, hd, p.rope_theta, &sn, &cs);
                const float y0 = x0 * cs - x1 * sn, y1 = x1 * cs + x0 * sn;
                if (hh < G) {
                    qs[hh * hd + e] = y0 * qscale;
                    qs[hh * hd + e + half] = y1 * qscale;
                } else {
                    const uint16_t b0 = f_to_bf16(y0), b1 = f_to_bf16(y1);
                    kn[e] = bf16_to_f(b0);
                    kn[e + half] = bf16_to_f(b1);
                    if (c == 0) {
                        kd[e] = b0;
                        kd[e + half] = b1;
                    }
                }
            }
            if (i < hd) {
                const uint16_t vb = f_to_bf16(xv[4 + k]);
                vn[i] = bf16_to_f(vb);
                if (c == 0)
                    vd[i] = vb;
            }
        }
    }
    consumer_bar();
    if (*reinterpret_cast<volatile int *>(s.flags))
        return false;
    // lane layout: lph lanes per head hold E = hd / lph of its elements; the
    // G heads of the group take lph * G lanes, and the warp's 32 lanes hold
    // PG such groups, each scoring a different position at the same time.
    // Lane li of a head holds, for E >= 8, the 8-element pieces (k lph + li)
    // (so that 8 neighbouring lanes read 128 contiguous bytes of a row, free
    // of bank conflicts), else elements [li E, li E + E).
    const int PG = p.att_pg;
    const int pg = lane / (lph * G), jh = (lane / lph) % G, li = lane % lph;
    const bool active = pg < PG;
    auto elem = [&](int k) { return E >= 8 ? ((k / 8) * lph + li) * 8 + (k % 8) : li * E + k; };
    // E bf16 values of the lane from the row at shared address row
    auto ldrow = [&](uint32_t row, float(&out)[E]) {
        if constexpr (E >= 8) {
#pragma unroll
            for (int c8 = 0; c8 < E / 8; ++c8) {
                float t[8];
                lds_bf16<8>(row + (uint32_t)((c8 * lph + li) * 16), t);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    out[c8 * 8 + u] = t[u];
            }
        } else {
            lds_bf16<E>(row + (uint32_t)(li * E * 2), out);
        }
    };
    float q[E], o[E];
    float m = -INFINITY, lsum = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        q[e] = active ? qs[jh * hd + elem(e)] : 0.f;
        o[e] = 0.f;
    }
    bool fail = false;
    uint64_t tA = 0, tB = 0;
    const int gstride = kConsumerWarps * PG;  // positions between a group's batches
    for (int i = 0; i < g.nchunks; ++i) {
        if (wt)
            tA = gtimer();
        if (!wait_full(p, s, kc)) {
            fail = true;
            break;
        }
        if (wt) {
            tB = gtimer();
            wt[0] += tB - tA;
        }
        const uint32_t ka = s.ring_a + (uint32_t)kc.st * p.stage_bytes;
        const uint32_t va = ka + (uint32_t)g.P * hd * 2;
        const int a = g.pa + i * g.P;
        const int n = min(g.P, g.pb - a);
        // four positions per group at a time (4 PG per warp): independent dot
        // products and shuffle reductions, then one online-softmax update
        for (int j0 = warp; j0 < n; j0 += 4 * gstride) {
            float sc[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int j = j0 + kConsumerWarps * pg + b * gstride;
                float kv_[E];
                ldrow(ka + (uint32_t)(j < n ? j : j0) * hd * 2, kv_);
                float d_ = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e)
                    d_ = fmaf(q[e], kv_[e], d_);
                sc[b] = d_;
            }
            for (int off = lph >> 1; off > 0; off >>= 1) {
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    sc[b] += __shfl_xor_sync(0xffffffffu, sc[b], off);
            }
            float mn = m;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                if (!active || j0 + kConsumerWarps * pg + b * gstride >= n)
                    sc[b] = -INFINITY;
                mn = fmaxf(mn, sc[b]);
            }
            if (mn == -INFINITY)  // this group has no position in the batch
                continue;
            const float corr = __expf(m - mn);
            float pr[4];
            lsum *= corr;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                pr[b] = __expf(sc[b] - mn);
                lsum += pr[b];
            }
#pragma unroll
            for (int e = 0; e < E; ++e)
                o[e] *= corr;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int j = j0 + kConsumerWarps * pg + b * gstride;
                if (active && j < n) {
                    float vv[E];
                    ldrow(va + (uint32_t)j * hd * 2, vv);
#pragma unroll
                    for (int e = 0; e < E; ++e)
                        o[e] = fmaf(pr[b], vv[e], o[e]);
                }
            }
            m = mn;
        }
        release_stage(p, s, kc, lane);
        kc.advance(p.ring_stages);
        if (wt)
            wt[1] += gtimer() - tB;
    }
    if (fail && lane == 0)
        s.flags[0] = 1;
    consumer_bar();
    if (*reinterpret_cast<volatile int *>(s.flags))
        return false;
    if (g.j0 <= p.pos && p.pos < g.j1 && warp == 0) {
        // the new position: K and V rows of this step (bf16 values as
        // floats), taken by position group 0
        float sc = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e)
            sc = fmaf(q[e], kn[elem(e)], sc);
        for (int off = lph >> 1; off > 0; off >>= 1)
            sc += __shfl_xor_sync(0xffffffffu, sc, off);
        if (pg == 0) {
            const float mn = fmaxf(m, sc);
            const float corr = __expf(m - mn);
            const float pr = __expf(sc - mn);
            lsum = lsum * corr + pr;
#pragma unroll
            for (int e = 0; e < E; ++e)
                o[e] = o[e] * corr + pr * vn[elem(e)];
            m = mn;
        }
    }
    // merge the position groups of the warp into group 0, as a tree: group
    // pg takes group pg + st (lanes st lph G further on hold the same head
    // elements) when pg is a multiple of 2 st; a group that saw no position
    // has m = -inf, l = 0
    for (int st = 1; st < PG; st <<= 1) {
        const int src = min(lane + st * lph * G, 31);
        const bool take = active && pg % (2 * st) == 0 && pg + st < PG;
        const float m2 = __shfl_sync(0xffffffffu, m, src);
        const float l2 = __shfl_sync(0xffffffffu, lsum, src);
        float ob[E];
#pragma unroll
        for (int e = 0; e < E; ++e)
            ob[e] = __shfl_sync(0xffffffffu, o[e], src);
        if (take) {
            const float mn = fmaxf(m, m2);
            const float fa = m == -INFINITY ? 0.f : __expf(m - mn);
            const float fb = m2 == -INFINITY ? 0.f : __expf(m2 - mn);
            lsum = lsum * fa + l2 * fb;
#pragma unroll
            for (int e = 0; e < E; ++e)
                o[e] = o[e] * fa + ob[e] * fb;
            m = mn;
        }
    }
    // per-warp state -> ws[w][jh][hd + 2]
    float *mine = ws + (size_t)warp * G * (hd + 2);
    if (pg == 0) {
#pragma unroll
        for (int e = 0; e < E; ++e)
            mine[jh * (hd + 2) + 2 + elem(e)] = o[e];
        if (li == 0) {
            mine[jh * (hd + 2) + 0] = m;
            mine[jh * (hd + 2) + 1] = lsum;
        }
    }
    consumer_bar();
    // the only non-empty chunk of the step writes the normalised output of
    // its heads directly; otherwise the partial (m, l, o) for the merge
    const bool direct = g.j0 == 0 && g.j1 == p.pos + 1;
    float *out = p.part + ((((size_t)l * nkv + gi) * p.attn_splits + c) * G) * (hd + 2);
    uint64_t *fin = p.attn + (size_t)l * nh * hd + (size_t)gi * G * hd;
    for (int i = ct; i < G * hd; i += kConsumerThreads) {
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
        if (direct) {
            fw_st(fin + i, O / L, otag);
            continue;
        }
        out[(size_t)hh * (hd + 2) + 2 + e] = O;
        if (e == 0) {
            out[(size_t)hh * (hd + 2) + 0] = M;
            out[(size_t)hh * (hd + 2) + 1] = L;
        }
    }
    return true;
}

// Merge of split-K partials: out[i] = sum_c e^(m_c - M) o_c[e] / L with
// M = max_c m_c and L = sum_c e^(m_c - M) l_c over the non-empty chunks c,
// for the attention-output elements first + i, i < count (element = head *
// hd + e; count <= kMaxPerThread * 256).  Thread t owns i = t + 256 j, in
// batches of B; for a batch the
// (m, l, o) of up to K chunks are loaded at once (one L2 round trip) and
// merged online in registers; address math is done once per element.
// K = 1 serves a single non-empty chunk (short contexts: out = o / l).
template <int K, int B>
__device__ __forceinline__ void merge_batches(const KParams &p, const float *part, int nne,
                                              int first, int count, uint64_t *out, int ct,
                                              uint32_t otag)
{
    const int hd = p.head_dim, G = p.group, C = p.attn_splits;
    const size_t cstride = (size_t)G * (hd + 2);  // chunk c + 1 of a head is this far on
    for (int j0 = 0; j0 < kMaxPerThread; j0 += B) {
        if (ct + j0 * kConsumerThreads >= count)
            break;
        const float *rp[B];  // (m, l, o[hd]) record of the element's head in chunk 0
        int eo[B];
        float M[B], L[B], O[B];
#pragma unroll
        for (int j = 0; j < B; ++j) {
            const int i = ct + (j0 + j) * kConsumerThreads;
            rp[j] = nullptr;
            eo[j] = 0;
            if (i < count) {
                const int h = (first + i) / hd;
                rp[j] = part + ((size_t)(h / G) * C * G + (h % G)) * (hd + 2);
                eo[j] = 2 + (first + i - h * hd);
            }
            M[j] = -INFINITY;
            L[j] = 0.f;
            O[j] = 0.f;
        }
        for (int c0 = 0; c0 < nne; c0 += K) {
            float2 ml[K][B];
            float oc[K][B];
#pragma unroll
            for (int k = 0; k < K; ++k)
#pragma unroll
                for (int j = 0; j < B; ++j) {
                    ml[k][j] = make_float2(-INFINITY, 0.f);
                    oc[k][j] = 0.f;
                    if (rp[j] && c0 + k < nne) {
                        const float *r = rp[j] + (c0 + k) * cstride;
                        ml[k][j] = __ldcg(reinterpret_cast<const float2 *>(r));
                        oc[k][j] = __ldcg(r + eo[j]);
                    }
                }
            if constexpr (K == 1) {
#pragma unroll
                for (int j = 0; j < B; ++j) {
                    L[j] = ml[0][j].y;
                    O[j] = oc[0][j];
                }
            } else {
#pragma unroll
                for (int k = 0; k < K; ++k)
#pragma unroll
                    for (int j = 0; j < B; ++j) {
                        if (rp[j] && c0 + k < nne) {
                            const float Mn = fmaxf(M[j], ml[k][j].x);
                            const float a = __expf(M[j] - Mn), b = __expf(ml[k][j].x - Mn);
                            L[j] = L[j] * a + ml[k][j].y * b;
                            O[j] = O[j] * a + oc[k][j] * b;
                            M[j] = Mn;
                        }
                    }
            }
        }
#pragma unroll
        for (int j = 0; j < B; ++j) {
            const int i = ct + (j0 + j) * kConsumerThreads;
            if (i < count)
                fw_st(out + i, O[j] / L[j], otag);
        }
    }
}

// Attention task (KV head g, chunk c): its partial, then the arrival.  With
// a single non-empty chunk (pos < chunk length) that chunk writes the output
// itself.  Otherwise each non-empty chunk task of (layer, g) adds one to the
// group's arrival counter with an acquire-release atomic behind its partial
// stores (the barrier before it makes them the CTA's, the release makes
// them visible first); the task that brings the count to this step's total
// merges the group's partials into the attention output of its G heads (its
// acquire orders those loads after every other chunk's stores).  The host
// counts the arrivals each step expects: arrive_base + nne.
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t *p, uint32_t v)
{
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;"
                 : "=r"(old)
                 : "l"(p), "r"(v)
                 : "memory");
    return old;
}

template <int E>
__device__ __forceinline__ bool attn_task(const KParams &p, const SmemLayout &s,
                                          const TaskDesc &d, const Geom &g, RingPos &kc,
                                          int ct, int warp, int lane, uint64_t *wt, uint32_t otag)
{
    if (!attn_chunk<E>(p, s, d, g, kc, ct, warp, lane, wt, otag))
        return false;
    const int l = d.layer, gi = d.r0, C = p.attn_splits;
    const int n = p.pos + 1;
    const int chunk = p.att_chunk;
    const int nne = (n + chunk - 1) / chunk;  // non-empty chunks: 0 .. nne-1
    if (nne == 1 || g.j1 <= g.j0)
        return true;  // written directly, or empty
    consumer_bar();  // every partial store of this task is issued
    int *last = s.flags + 1;
    if (ct == 0) {
        const uint32_t old = atom_add_acq_rel(p.arrive + (size_t)l * p.n_kv_heads + gi, 1u);
        *last = old == p.arrive_base + (uint32_t)(nne - 1);
    }
    consumer_bar();
    if (*reinterpret_cast<volatile int *>(last)) {
        const int hd = p.head_dim, G = p.group, N = p.n_heads * hd;
        const float *part = p.part + (size_t)l * p.n_kv_heads * C * G * (hd + 2);
        uint64_t *out = p.attn + (size_t)l * N + (size_t)gi * G * hd;
        merge_batches<4, 4>(p, part, nne, gi * G * hd, G * hd, out, ct, otag);
    }
    return true;
}

// O-projection prologue of the position-0 schedule.  At position 0 the
// softmax runs over the single key of this step, so every weight is 1 and the
// attention output of head h is the V row of its KV head h / G as stored in
// the cache (bf16), and RoPE at angle 0 is the identity.  Cache row 0 (K = k,
// V = v, rounded to bf16) is written in shares: of its E = 2 nkv hd elements
// (K of every head, then V), the tile of rows [r0, r1) writes
// [r0 E / h, r1 E / h).
__device__ void pos0_prologue(const KParams &p, const SmemLayout &s, const TaskDesc &d, int ct)
{
    const int l = d.layer, hd = p.head_dim, nh = p.n_heads, nkv = p.n_kv_heads, G = p.group;
    const int KV = nkv * hd;  // elements of one of K, V
    const uint64_t *qkv = p.qkv + (size_t)l * p.qkv_rows;
    const uint64_t *ksrc = qkv + (size_t)nh * hd, *vsrc = ksrc + KV;
    // element r of V (KV head r / hd) is the output of the G heads of that
    // group: thread t takes r = t + 256 j, one flagged word and G stores each
    // and the tile's share of cache row 0: elements i = a + t + 256 k of
    // (K | V), the first two of them loaded together with the V words
    const int E = 2 * KV;
    const int a = (int)((int64_t)d.r0 * E / p.hidden), b = (int)((int64_t)d.r1 * E / p.hidden);
    const size_t blk = (size_t)p.max_ctx * hd;  // one (layer, K|V, head) block
    const uint64_t *sh[2];
    uint64_t shw[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int i = a + ct + k * kConsumerThreads;
        sh[k] = i < b ? ksrc + i : nullptr;
        shw[k] = sh[k] ? fw_ld(sh[k]) : 0ull;
    }
    float v[kMaxPerThread];
    bool ok = fw_read_strided<kMaxPerThread>(p, s, vsrc, KV, ct, v);
    for (int i0 = a + ct; i0 < b && ok; i0 += 2 * kConsumerThreads) {
        float kvv[2];
        if (i0 == a + ct && (!sh[0] || fw_ok(shw[0], p.tag)) && (!sh[1] || fw_ok(shw[1], p.tag))) {
            kvv[0] = fw_val(shw[0]);
            kvv[1] = fw_val(shw[1]);
        } else {
            const int i1 = i0 + kConsumerThreads;
            const uint64_t *w[2] = {ksrc + i0, i1 < b ? ksrc + i1 : nullptr};
            ok = fw_gather<2>(p, s, w, kvv);
        }
        for (int k = 0; k < 2 && ok; ++k) {
            const int i = i0 + k * kConsumerThreads;
            if (i >= b)
                break;
            const int which = i >= KV, r = i - which * KV;  // 0: K, 1: V
            const int g = r / hd, e = r - g * hd;
            p.kv[(((size_t)l * 2 + which) * nkv + g) * blk + e] = f_to_bf16(kvv[k]);
        }
    }
    if (!ok)
        s.flags[0] = 1;  // before the barrier below: every thread sees it after
#pragma unroll
    for (int j = 0; j < kMaxPerThread; ++j) {
        const int r = ct + j * kConsumerThreads;
        if (r < KV) {
            const int g = r / hd, e = r - g * hd;
            const float x = bf16_to_f(f_to_bf16(v[j]));
            for (int hh = 0; hh < G; ++hh)
                s.vec[vidx((g * G + hh) * hd + e)] = x;
        }
    }
    consumer_bar();
}

// O-projection prologue: the merged attention output of layer l -> vec
// (one L2 round trip).  n_heads * head_dim <= kMaxPerThread * 256.
__device__ void attn_prologue(const KParams &p, const SmemLayout &s, int l, int ct)
{
    const int N = p.n_heads * p.head_dim;
    const uint64_t *src = p.attn + (size_t)l * N;
    float v[kMaxPerThread];
    if (!fw_read_strided<kMaxPerThread>(p, s, src, N, ct, v))
        s.flags[0] = 1;  // before the barrier below: every thread sees it after
#pragma unroll
    for (int j = 0; j < kMaxPerThread; ++j) {
        const int i = ct + j * kConsumerThreads;
        if (i < N)
            s.vec[vidx(i)] = v[j];
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

// Fused FFN, after its gate/up GEMV: the slice's R SwiGLU activations
// act[j] = silu(gate_j) up_j are in vec[0, R) (int8 weights: also as int16
// pairs at byte kQOff of vec, with one scale for the slice in scr[8]); then
// the slice's columns of Wdown stream through the ring, 16-byte column group
// jb of chunk row lr at (jb nrows + lr) * 16 of the stage.  Thread t owns the
// rows t + 256 k of each chunk: it forms sum_j W[row][r0 + j] act[j] (times
// the row's int8 scale, loaded before the chunk's ring wait) and adds it
// into the layer's fixed-point residual.  The 16-byte pieces a warp reads at
// once are consecutive: free of bank conflicts.
constexpr int kQOff = 1024;  // byte offset of the int16 activation copy in vec

// bf16 weights: the activations stay in shared memory (broadcast loads),
// which measured faster than register copies for the narrow slices of the
// models that fuse the level
__device__ __forceinline__ bool ffn_down_bf16(const KParams &p, const SmemLayout &s,
                                              const Geom &g, const TaskDesc &d, RingPos &kc,
                                              int ct, int lane)
{
    constexpr int E = 8;  // bf16 elements per box row
    const int ncb = g.ncb, h = p.hidden;
    long long *acc_out = p.xacc + (size_t)d.layer * h;
    for (int c2 = 0; c2 < g.nck2; ++c2) {
        const int r0w = c2 * g.rpc2, nrows = min(g.rpc2, h - r0w);
        if (!wait_full(p, s, kc))
            return false;
        const uint32_t st_a = s.ring_a + (uint32_t)kc.st * p.stage_bytes;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int lr = ct + kConsumerThreads * k;
            if (lr < nrows) {
                f2_t acc = 0ull;
                for (int jb = 0; jb < ncb; ++jb) {
                    const WVec<16> w = ldw<16>(st_a + (uint32_t)((jb * nrows + lr) * 16));
                    f2_t x[E / 2];
#pragma unroll
                    for (int u = 0; u < E / 2; ++u) {
                        const uint2 t = lds64(s.vec_a + (uint32_t)(jb * E + 2 * u) * 4);
                        x[u] = pk2(__uint_as_float(t.x), __uint_as_float(t.y));
                    }
                    acc = vdot2<2, 16>(w, x, acc);
                }
                red_add_fix(acc_out + r0w + lr, to_fix(sum2(acc)));
            }
        }
        release_stage(p, s, kc, lane);
        kc.advance(p.ring_stages);
    }
    return true;
}

// int8 weights: every thread holds the slice's activations as int16 pairs
// (NCB >= ncb column groups of 16) and multiplies them with dp2a
template <int NCB>
__device__ __forceinline__ bool ffn_down_i8(const KParams &p, const SmemLayout &s, const Geom &g,
                                            const TaskDesc &d, RingPos &kc, int ct, int lane)
{
    const int ncb = g.ncb, h = p.hidden;
    long long *acc_out = p.xacc + (size_t)d.layer * h;
    uint32_t xq[NCB * 8];
#pragma unroll
    for (int jb = 0; jb < NCB; ++jb)
#pragma unroll
        for (int k = 0; k < 8; k += 4) {
            uint4 u = make_uint4(0u, 0u, 0u, 0u);
            if (jb < ncb)
                u = lds128(s.vec_a + kQOff + (uint32_t)(jb * 8 + k) * 4);
            xq[jb * 8 + k] = u.x;
            xq[jb * 8 + k + 1] = u.y;
            xq[jb * 8 + k + 2] = u.z;
            xq[jb * 8 + k + 3] = u.w;
        }
    const float xs = s.scr[8];
    for (int c2 = 0; c2 < g.nck2; ++c2) {
        const int r0w = c2 * g.rpc2, nrows = min(g.rpc2, h - r0w);
        float scl[16];  // rows per thread per chunk <= stage / (16 B * 256)
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int lr = ct + kConsumerThreads * k;
            scl[k] = (d.s2 && lr < nrows) ? fp16_to_f(__ldg(d.s2 + r0w + lr)) : 1.f;
        }
        if (!wait_full(p, s, kc))
            return false;
        const uint32_t st_a = s.ring_a + (uint32_t)kc.st * p.stage_bytes;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int lr = ct + kConsumerThreads * k;
            if (lr < nrows) {
                int acc[2] = {0, 0};
#pragma unroll
                for (int jb = 0; jb < NCB; ++jb) {
                    if (jb < ncb) {
                        const uint4 w = lds128(st_a + (uint32_t)((jb * nrows + lr) * 16));
                        const uint32_t A[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            acc[0] = dp2a_lo(xq[jb * 8 + 2 * q], A[q], acc[0]);
                            acc[1] = dp2a_hi(xq[jb * 8 + 2 * q + 1], A[q], acc[1]);
                        }
                    }
                }
                const float sum = (float)(acc[0] + acc[1]) * xs;
                red_add_fix(acc_out + r0w + lr, to_fix(sum * scl[k]));
            }
        }
        release_stage(p, s, kc, lane);
        kc.advance(p.ring_stages);
    }
    return true;
}

// The slice's activations into vec[0, R); for int8 weights also as int16
// pairs at vec + kQOff with their step in scr[8] (one scale for the slice:
// the largest |act| over 32767), then the dispatch on the column groups.
template <int Q8, int GENERIC>
__device__ __forceinline__ bool ffn_down(const KParams &p, const SmemLayout &s, const Geom &g,
                                         const TaskDesc &d, RingPos &kc, int ct, int lane,
                                         float sc0, float sc1)
{
    float a = 0.f;
    if (ct < g.R) {
        const float gt = row_total(s, g, ct) * sc0;
        const float up = row_total(s, g, g.R + ct) * sc1;
        a = gt / (1.f + __expf(-gt)) * up;
        s.vec[ct] = a;
    }
    const bool q8 = GENERIC ? g.esz == 1 : Q8 == 1;
    if (q8) {
        float m = fabsf(a);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((ct & 31) == 0)
            s.scr[ct >> 5] = m;
    }
    consumer_bar();
    if (q8) {
        float m = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w)
            m = fmaxf(m, s.scr[w]);
        const float inv = m > 0.f ? 32767.f / m : 0.f;
        if (ct < g.R) {
            const int q = max(-32767, min(32767, __float2int_rn(a * inv)));
            reinterpret_cast<short *>(reinterpret_cast<uint8_t *>(s.vec) + kQOff)[ct] = (short)q;
        }
        if (ct == 0)
            s.scr[8] = m * (1.f / 32767.f);
        consumer_bar();
    }
    const int ncb = g.ncb;
    if (g.esz == 1) {
        if constexpr (GENERIC || Q8 == 1) {
            if (ncb <= 2)
                return ffn_down_i8<2>(p, s, g, d, kc, ct, lane);
            if (ncb <= 4)
                return ffn_down_i8<4>(p, s, g, d, kc, ct, lane);
            return ffn_down_i8<8>(p, s, g, d, kc, ct, lane);
        }
    } else {
        if constexpr (GENERIC || Q8 == 0)
            return ffn_down_bf16(p, s, g, d, kc, ct, lane);
    }
    return false;
}

// ---------------------------------------------------------- consumer loop
template <int Q8, int ATT_E, int GENERIC, int FUSED>
__device__ __forceinline__ void consumer_loop(const KParams &p, const SmemLayout &s, int qb,
                                              int qe, int ct)
{
    const int warp = ct >> 5, lane = ct & 31;
    unsigned long long *prof =
        (p.prof && ct == 0) ? p.prof + (size_t)blockIdx.x * kProfKinds * kProfFields : nullptr;
    if (prof)
        prof[0] = gtimer();
    const bool wprof = p.prof != nullptr && lane == 0;
    uint64_t wt_store[2] = {0, 0};
    uint64_t *wt = wprof ? wt_store : nullptr;
    RingPos kc{0u, 0, 0u};  // chunks consumed
    int token = -1;
    if (ct == 0 && qb < qe)
        stage_task(s.ctask_a, p.tasks + qb);
    for (int ti = qb; ti < qe; ++ti) {
        const uint32_t slot = s.ctask_a + ((ti - qb) & 1) * sizeof(TaskDesc);
        if (ct == 0) {
            stage_task_wait();  // record of task ti (issued one task ago)
            s.flags[2] = ti;    // for the error record of a flagged read that gives up
        }
        consumer_bar();
        const TaskDesc d = read_staged(slot);
        uint64_t t_w0 = 0, t_w1 = 0, t_pro = 0, t_epi = 0;
        if (prof) {
            t_w0 = gtimer();
            s.wacc[0] = s.wacc[1] = 0ull;
            *reinterpret_cast<volatile unsigned long long *>(s.flags + 4) = 0ull;
        }
        if (wprof)
            wt_store[0] = wt_store[1] = 0;
        // loads that do not depend on this step's activations go out before
        // the task's wait: the RMSNorm gains and the int8 row scales of the
        // epilogue (thread t finalises row r0 + t; R <= 256)
        const Geom g = task_geom(p, d);
        // (kept as raw bits until first use: a conversion here would wait for
        // the loads before the task's own wait starts)
        uint32_t gv[kMaxPerThread];
        const bool norm = d.kind == TK_QKV || d.kind == TK_GATEUP || d.kind == TK_FFN ||
                          d.kind == TK_LMHEAD;
#pragma unroll
        for (int j = 0; j < kMaxPerThread; ++j) {
            const int i = ct + j * kConsumerThreads;
            gv[j] = (norm && i < p.hidden) ? (uint32_t)__ldg(d.gain + i) : 0u;
        }
        uint32_t sc0r = 0x3c00u, sc1r = 0x3c00u;  // fp16 1.0
        if (d.kind != TK_ATTN && ct < g.R) {
            if (d.s0)
                sc0r = __ldg(d.s0 + ct);
            if (d.s1)
                sc1r = __ldg(d.s1 + ct);
        }
        if (ct == 0) {
            if (ti + 1 < qe)  // the slot read at ti - 1 is free again (barrier above)
                stage_task(s.ctask_a + ((ti + 1 - qb) & 1) * sizeof(TaskDesc), p.tasks + ti + 1);
            // with flagged waits the task's reads of its flagged inputs are
            // its wait (every input of every task is flagged then)
            if (!p.flagged && !wait_counter(p, d, ti))
                s.flags[0] = 1;
        }
        consumer_bar();
        if (*reinterpret_cast<volatile int *>(s.flags))
            break;
        // the tag of this task's flagged outputs (the test hook that withholds
        // a task's signal gives them a wrong one)
        const uint32_t otag =
            (p.flagged && ti == p.skip_signal_task) ? p.tag ^ 0x80000000u : p.tag;
        if (prof)
            t_w1 = gtimer();
        const int l = d.layer;
        bool ok = true;
        if (d.kind == TK_ATTN) {
            if constexpr (!GENERIC) {
                ok = attn_task<ATT_E>(p, s, d, g, kc, ct, warp, lane, wt, otag);
            } else {
                switch (p.att_e) {
                case 1: ok = attn_task<1>(p, s, d, g, kc, ct, warp, lane, wt, otag); break;
                case 2: ok = attn_task<2>(p, s, d, g, kc, ct, warp, lane, wt, otag); break;
                case 4: ok = attn_task<4>(p, s, d, g, kc, ct, warp, lane, wt, otag); break;
                case 8: ok = attn_task<8>(p, s, d, g, kc, ct, warp, lane, wt, otag); break;
                default: ok = attn_task<16>(p, s, d, g, kc, ct, warp, lane, wt, otag); break;
                }
            }
            if (prof)
                t_pro = t_epi = gtimer();
        } else {
            // prologue -> s.vec (one call site per prologue kind: the kernel
            // is one persistent program, and its instruction footprint counts)
            if (norm) {
                // the RMSNorm input: the embedding row (layer 0), the previous
                // layer's residual (fixed point after a fused FFN level), or
                // the residual after attention (gate/up, fused FFN)
                const uint64_t *xw = nullptr;
                const uint16_t *xb = nullptr;
                const long long *xq = nullptr;
                const int lp = d.kind == TK_LMHEAD ? p.n_layers - 1 : l - 1;
                if (d.kind == TK_GATEUP || d.kind == TK_FFN) {
                    xw = p.xmid + (size_t)l * p.hidden;
                } else if (d.kind == TK_QKV && l == 0) {
                    if (token < 0)
                        token = resolve_token(p);
                    xb = p.embed + (size_t)token * p.hidden;
                } else if (p.ffn_fused) {
                    xq = p.xacc + (size_t)lp * p.hidden;
                } else {
                    xw = p.xout + (size_t)lp * p.hidden;
                }
                rmsnorm_prologue(p, s, xw, xb, xq, gv, ct);
            } else if (d.kind == TK_OPROJ) {
                if (d.flags & TF_POS0)
                    pos0_prologue(p, s, d, ct);
                else
                    attn_prologue(p, s, l, ct);
            }
            // (DOWN has no prologue: each warp loads its slice of the SwiGLU
            // activations from the flagged words straight into registers)
            // a prologue that gave up raised the abort flag before its last
            // barrier (DOWN has none, and nothing since its wait raised it)
            if (*reinterpret_cast<volatile int *>(s.flags))
                break;
            // residual inputs of the epilogue: their loads go out now and are
            // used after the GEMV (thread t owns output row r0 + t; R <= 256);
            // a flagged one is checked (and polled again if need be) there
            float base = 0.f;
            const uint64_t *bsrc = nullptr;
            uint64_t bw = 0;
            if (ct < g.R) {
                const int r = d.r0 + ct;
                if (d.kind == TK_OPROJ) {
                    if (l == 0) {
                        if (token < 0)
                            token = resolve_token(p);
                        base = bf16_to_f(__ldg(p.embed + (size_t)token * p.hidden + r));
                    } else if (p.ffn_fused) {
                        base = from_fix(__ldcg(p.xacc + (size_t)(l - 1) * p.hidden + r));
                    } else {
                        bsrc = p.xout + (size_t)(l - 1) * p.hidden + r;
                    }
                } else if (d.kind == TK_DOWN) {
                    bsrc = p.xmid + (size_t)l * p.hidden + r;
                }
                if (bsrc)
                    bw = fw_ld(bsrc);
            }
            if (prof)
                t_pro = gtimer();
            ok = run_gemv<Q8, GENERIC>(p, s, g, kc, warp, lane,
                          d.kind == TK_DOWN ? p.act + (size_t)l * p.ffn : nullptr, wt);
            if (!ok && lane == 0) {
                record_error(p, 2u, ti, -1, 0u, 0u);
                s.flags[0] = 1;
            }
            consumer_bar();
            if (prof)
                t_epi = gtimer();
            ok = *reinterpret_cast<volatile int *>(s.flags) == 0;
            const float sc0 = fp16_to_f((uint16_t)sc0r), sc1 = fp16_to_f((uint16_t)sc1r);
            if (ok && bsrc) {
                if (fw_ok(bw, p.tag)) {
                    base = fw_val(bw);
                } else {
                    const uint64_t *const a1[1] = {bsrc};
                    float v1[1];
                    ok = fw_gather<1>(p, s, a1, v1);
                    base = v1[0];
                }
            }
            if (ok) {
                // epilogue: thread t finalises output row r0 + t
                if (d.kind == TK_QKV) {
                    const int off = d.mat == 0 ? 0
                                    : d.mat == 1 ? p.n_heads * p.head_dim
                                                 : (p.n_heads + p.n_kv_heads) * p.head_dim;
                    uint64_t *out = p.qkv + (size_t)l * p.qkv_rows + off + d.r0;
                    for (int t = ct; t < g.R; t += kConsumerThreads)
                        fw_st(out + t, row_total(s, g, t) * sc0, otag);
                } else if (d.kind == TK_OPROJ) {
                    if (ct < g.R) {
                        const float v = base + row_total(s, g, ct) * sc0;
                        fw_st(p.xmid + (size_t)l * p.hidden + d.r0 + ct, v, otag);
                        if (p.ffn_fused)  // the FFN slices add into this
                            p.xacc[(size_t)l * p.hidden + d.r0 + ct] = to_fix(v);
                    }
                } else if (d.kind == TK_FFN) {
                    if constexpr (FUSED || GENERIC)
                        ok = ffn_down<Q8, GENERIC>(p, s, g, d, kc, ct, lane, sc0, sc1);
                } else if (d.kind == TK_GATEUP) {
                    for (int t = ct; t < g.R; t += kConsumerThreads) {
                        const float gt = row_total(s, g, t) * sc0;
                        const float up = row_total(s, g, g.R + t) * sc1;
                        const float silu = gt / (1.f + __expf(-gt));
                        fw32_st(p.act + (size_t)l * p.ffn + d.r0 + t, silu * up, fw8_tag(otag));
                    }
                } else if (d.kind == TK_DOWN) {
                    if (ct < g.R)
                        fw_st(p.xout + (size_t)l * p.hidden + d.r0 + ct,
                              base + row_total(s, g, ct) * sc0, otag);
                } else {  // TK_LMHEAD
                    unsigned long long best = 0ull;
                    for (int t = ct; t < g.R; t += kConsumerThreads) {
                        const float y = row_total(s, g, t) * sc0;
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
                    if (ct == 0) {
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
        if (wprof) {
            atomicAdd(&s.wacc[0], (unsigned long long)wt_store[0]);
            atomicAdd(&s.wacc[1], (unsigned long long)wt_store[1]);
        }
        consumer_bar();
        if (*reinterpret_cast<volatile int *>(s.flags))
            break;
        // release: the CTA barrier above orders every thread's stores before
        // this release-add (cumulativity), so the waiters' acquire sees them.
        // With flagged waits nobody waits on the level counters.
        if (ct == 0 && !p.flagged && d.signal_ctr >= 0 && ti != p.skip_signal_task)
            red_release_add(p.counters + d.signal_ctr, 1u);
        if (prof) {
            const uint64_t t_end = gtimer();
            unsigned long long *pk = prof + (size_t)d.kind * kProfFields;
            // the flagged polls of a task happen in its prologue (attention:
            // its tile), except DOWN's, which its GEMV warps make
            const uint64_t fw = *reinterpret_cast<volatile unsigned long long *>(s.flags + 4);
            pk[0] += 1;
            pk[1] += t_w1 - t_w0;
            pk[2] += t_pro - t_w1 - (d.kind == TK_DOWN ? 0ull : min(fw, t_pro - t_w1));
            pk[3] += fw;
            pk[4] += t_end - t_w1;
            pk[5] += t_end - t_epi;
            pk[6] += s.wacc[0];
            pk[7] += s.wacc[1];
        }
    }
    if (prof)
        prof[1] = gtimer();
}

// ------------------------------------------------------------------- kernel
// One fast instance per (weight format, attention lane width), holding only
// the paths its models use, plus one generic instance for the rest.
template <int Q8, int ATT_E, int GENERIC, int FUSED>
__global__ void __launch_bounds__(kThreads, 1) amk_decode_kernel(const __grid_constant__ KParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const SmemLayout s = smem_layout(smem_raw, p);
    const int tid = threadIdx.x;
    const int qb = p.queue_off[blockIdx.x], qe = p.queue_off[blockIdx.x + 1];

    if (tid == 0) {
        for (int i = 0; i < p.ring_stages; ++i) {
            for (int pc = 0; pc < kPieces; ++pc)
                mbar_init(s.full_a + 8 * (i * kPieces + pc), 1);
            mbar_init(s.empty_a + 8 * i, kConsumerWarps);
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
    if (tid < kProducerThreads) {
        setmaxnreg_dec<kProducerRegs>();
        if (tid == 0)
            producer_loop(p, s, qb, qe);
        return;
    }
    setmaxnreg_inc<kConsumerRegs>();
    consumer_loop<Q8, ATT_E, GENERIC, FUSED>(p, s, qb, qe, tid - kProducerThreads);
    // On abort the producer notices the flag, drains its copies and returns.
}

}  // namespace

}  // namespace amk
