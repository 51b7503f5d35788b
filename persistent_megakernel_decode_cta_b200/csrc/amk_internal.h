// amk_internal.h -- structures shared by the host lowering/launcher and the
// sm_100a megakernel.  Plain PODs: the host writes them once at create time
// and the kernel reads them.
#ifndef AMK_INTERNAL_H
#define AMK_INTERNAL_H

#include <stdint.h>

#include <cuda_runtime.h>

#include "amk.h"

#ifdef __cplusplus
extern "C" {
#endif
// Records a thread-local error message and returns `code`.
int amk_set_error(int code, const char *fmt, ...);
#ifdef __cplusplus
}
#endif

namespace amk {

// Persistent CTA shape: one producer warpgroup (lane 0 of its first warp
// issues the TMA bulk copies; the warpgroup drops to kProducerRegs registers)
// and two consumer warpgroups = 8 compute warps (raised to kConsumerRegs).
// 128 * 56 + 256 * 224 = 384 * 168: the split uses exactly the registers the
// block is launched with.
constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kProducerThreads = 128;
constexpr int kThreads = kProducerThreads + kConsumerThreads;
constexpr int kLaunchRegs = 168;
constexpr int kProducerRegs = 56;
constexpr int kConsumerRegs = 224;
static_assert(kProducerThreads * kProducerRegs + kConsumerThreads * kConsumerRegs ==
                  kThreads * kLaunchRegs, "register split must equal the launch budget");
constexpr int kMaxTaskRows = 256;   // output rows of one GEMV task (red buffer)
// Positions of a split-K attention chunk: ceil(n / attn_splits) for n
// positions, but at least kMinAttnChunk, so that short contexts use fewer,
// longer chunks (the kernel and the host's arrival count both use this).
constexpr int kMinAttnChunk = 32;
// W4A16 weights: inputs per fp16 scale, and the bytes of one packed row of K
// inputs as the ring streams it: K / 2 code bytes (input 2i in the low nibble
// of byte i, 4-bit two's complement), then the row's ceil(K / 128) scales,
// zero-padded to a multiple of 16 bytes.
constexpr int kQ4Group = 128;
inline __host__ __device__ int q4_row_bytes(int K)
{
    return (K / 2 + 2 * ((K + kQ4Group - 1) / kQ4Group) + 15) & ~15;
}
inline __host__ __device__ int attn_chunk_len(int n, int splits)
{
    const int c = (n + splits - 1) / splits;
    return c > kMinAttnChunk ? c : kMinAttnChunk;
}
constexpr int kMaxStages = 16;
// A ring stage's copy goes out in up to kPieces pieces of about KParams::piece bytes,
// each completing on its own mbarrier, so that the producer can keep a
// bounded number of bytes in flight (KParams::inflight).
constexpr int kPieces = 4;
constexpr int kPieceQueue = 32;     // pieces the producer tracks at once

// Task kinds (the instruction set: GEMV row tiles with fused prologues and
// epilogues, and the split-K attention tile).
enum TaskKind : uint8_t {
    TK_QKV = 1,     // rows of Wq|Wk|Wv (mat 0/1/2), RMSNorm prologue, raw q/k/v out
    TK_ATTN = 2,    // (kv head g, split c): RoPE, KV append (c == 0), partial softmax;
                    // the head's last chunk to finish merges all of them
    TK_OPROJ = 3,   // rows of Wo, attention-output prologue, residual epilogue
    TK_GATEUP = 4,  // rows of Wgate and Wup, RMSNorm prologue, SwiGLU epilogue
    TK_DOWN = 5,    // rows of Wdown, residual epilogue
    TK_LMHEAD = 6,  // rows of the LM head, final RMSNorm prologue, argmax epilogue
    TK_FFN = 7,     // FFN slice [r0, r1): RMSNorm prologue, rows of Wgate and Wup, SwiGLU,
                    // then the columns [r0, r1) of Wdown (2-D TMA boxes); the partial
                    // down projection is added into the layer's fixed-point residual
};

enum TaskFlags : uint8_t {
    TF_RESET_ARGKEY = 1,  // this task clears the next step's argmax key
    TF_POS0 = 2,          // O-projection of the position-0 schedule: head outputs = V rows,
                          // and the task writes its share of KV-cache row 0
};

struct TaskDesc {           // 96 bytes, read-only for the kernel
    uint8_t kind, mat, flags, pad;
    int32_t layer;
    int32_t wait_ctr;       // -1: no wait
    uint32_t wait_count;    // threshold t within one epoch
    uint32_t wait_total;    // producers of wait_ctr (signals per epoch)
    int32_t signal_ctr;     // -1: no signal
    int32_t r0, r1;         // GEMV: output rows [r0, r1); ATTN: r0 = kv head g, r1 = chunk c
    // resolved by the host once the weights are known:
    const void *w0, *w1;    // GEMV: row r0 of part 0 / part 1 (gate/up); ATTN: K / V cache
                            //   block of (layer, g)
    const uint16_t *s0, *s1;  // fp16 row scales at row r0 (W8A16), or null
    const uint16_t *gain;     // RMSNorm gain of the prologue, or null
    const uint16_t *s2;       // TK_FFN: fp16 row scales of Wdown [hidden] (W8A16), or null
    // ring geometry of a GEMV task (zero for ATTN), computed by the host when it
    // resolves the task (amk_task_geometry), so that neither the producer nor
    // the consumers divide by run-time values at a task boundary:
    uint16_t nchunks;         // ring chunks: the row GEMV's, then a fused FFN's Wdown ones
    uint16_t ngu;             // chunks of the row GEMV (of all its parts)
    uint16_t rpc;             // rows per chunk (a multiple of the row groups and of the
                              //   16-byte granule of the row length)
    uint16_t nck;             // chunks per part (gate and up are two parts)
    uint16_t rpc2, nck2;      // fused FFN Wdown: rows per chunk, chunks
    uint16_t ncb;             // fused FFN Wdown: 16-byte column groups of the slice
    uint8_t ks_log2, rg_log2; // the 8 consumer warps: 2^ks K-slices x 2^rg row groups
};
static_assert(sizeof(TaskDesc) == 96, "TaskDesc is 96 bytes (six 16-byte pieces)");

// Per-layer weight pointers (device copies of the caller's pointers).
struct LayerPtrs {
    const void *w[7];          // 0 q, 1 k, 2 v, 3 o, 4 gate, 5 up, 6 down
    const uint16_t *s[7];      // fp16 row scales (W8A16) or null
    const uint16_t *attn_norm, *ffn_norm;
};
enum { W_Q = 0, W_K, W_V, W_O, W_GATE, W_UP, W_DOWN };

struct ErrorWord {
    uint32_t code;      // 0 = ok, 1 = counter wait timeout, 2 = ring wait timeout
    int32_t task, counter, sm;
    uint32_t seen, target;
    uint32_t pad[2];
};

struct KParams {
    // schedule
    const TaskDesc *tasks;     // grouped by SM, in queue order
    const int32_t *queue_off;  // [n_sms + 1]
    uint32_t *counters;
    uint32_t *arrive;          // [L][nkv]: attention chunk tasks arrived, monotonic
    ErrorWord *err;
    // weights (the per-task pointers live in the task records)
    const uint16_t *embed;
    // state and activations.  The vectors one level hands to the next are
    // flagged words: 64 bits each, the fp32 value in the low half and the tag
    // of the step that wrote it in the high half (see fw_st in the kernel)
    uint64_t *qkv;    // [L][qkv_rows]: q | k | v, before RoPE (flagged)
    float *part;      // [L][nkv][C][G][hd + 2]: split-K partials (m, l, o[hd])
    uint64_t *attn;   // [L][nh * hd]: attention output, the chunks merged (flagged)
    uint64_t *xmid;   // [L][h]: residual after attention (flagged)
    uint64_t *xout;   // [L][h]: residual after the FFN (flagged)
    uint32_t *act;    // [L][ffn]: SwiGLU activations, 32-bit flagged words (the fp32
                      // value's low 8 bits replaced by the step's 8-bit tag)
    long long *xacc;  // [L][h]: residual after the FFN in fixed point (value * 2^32), when
                      // the FFN level is fused: OPROJ writes the residual, FFN slices add
    const void *dmaps;  // [L] 128-byte tensor maps of Wdown (fused FFN), 64-byte aligned
    const uint8_t *dpack;  // fused FFN: Wdown of every layer packed in 16-byte column
                           // groups, [L][ffn * esz / 16][hidden][16 B], or null: the
                           // tensor maps read the caller's Wdown
    float *logits;    // [vocab]
    unsigned long long *argkey;  // [2] packed (ordered logit << 32 | ~index)
    uint16_t *kv;     // bf16 [L][2][nkv][max_ctx][hd]
    // shapes
    int32_t hidden, n_layers, n_heads, n_kv_heads, head_dim, ffn, vocab, max_ctx;
    int32_t qkv_rows, group, attn_splits, quant, tied;
    float rms_eps, rope_theta;
    // ring
    int32_t ring_stages, stage_bytes, vec_floats;
    // attention lane layout
    int32_t att_lph, att_hpb, att_e;  // lanes per head, heads per batch, elems per lane
    int32_t att_pg;                   // position groups per warp (lph * G lanes each)
    int32_t generic;            // 1: run the generic kernel instance
    int32_t ffn_fused, ffn_box_rows;
    // step
    int32_t pos, token;         // token < 0: previous step's argmax
    uint32_t epoch;             // steps since reset (counter targets)
    uint32_t arrive_base;       // attention arrivals of earlier steps per (layer, kv head)
    int32_t parity;             // epoch & 1
    uint64_t timeout_ns;
    uint32_t lookahead;         // L2 prefetch distance past the ring copies (bytes), 0 = off
    uint32_t inflight;          // cap on bulk-copy bytes in flight per SM (0xffffffff: none)
    uint32_t piece;             // bytes of a copy piece (multiple of 16)
    int32_t att_chunk;          // positions per split-K attention chunk at this step
    int32_t att_P;              // KV positions per ring stage (stage_bytes / (4 head_dim))
    int32_t skip_signal_task;   // test hook, -1 = off (with flagged waits: that task's
                                // flagged words carry a wrong tag)
    uint32_t tag;               // this step's tag in the flagged words (never 0)
    int32_t flagged;            // 1: tasks wait on the flagged words they read instead of
                                // level counters, and signal no counter (FFN levels split)
    unsigned long long *prof;   // [n_sms][kProfKinds][kProfFields] phase timers, or null
};
constexpr int kProfKinds = AMK_PROF_KINDS;
constexpr int kProfFields = AMK_PROF_FIELDS;

}  // namespace amk

#endif
