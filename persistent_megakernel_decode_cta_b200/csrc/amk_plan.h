// amk_plan.h -- the lowered schedule of one decode step (host side).
#ifndef AMK_PLAN_H
#define AMK_PLAN_H

#include <cstdint>
#include <vector>

#include "amk.h"
#include "amk_internal.h"

struct amk_plan {
    amk_config cfg;
    amk_options opt;       // effective knobs (ring_stages, attn_splits resolved)
    int n_sms = 0;
    int group = 0, qkv_rows = 0, vec_floats = 0, smem_bytes = 0;
    int att_lph = 0, att_hpb = 0, att_e = 0;
    int generic = 0;  // 1: odd row widths or a bf16 tied head on int8 layers
    std::vector<amk::TaskDesc> tasks;  // grouped by SM, queue order
    std::vector<int32_t> queue_off;    // [n_sms + 1]
    int n_counters = 0;  // level counters (the validator's graph)
    int n_arrive = 0;    // attention arrival counters, [L][nkv], after them
    int att_pg = 1;      // attention position groups per warp
    int ffn_fused = 0;   // 1: one FFN level per layer (gate/up + down column slice)
    int flagged = 0;     // 1: tasks wait on the flagged words they read, not on counters
    int ffn_box_rows = 0;  // rows of a Wdown TMA box (divides hidden)
    int is_pos0 = 0;     // 1: the schedule of steps at position 0 (no attention level)
    amk_plan *pos0 = nullptr;  // owned: that schedule, for a plan of all other steps
    uint64_t uid = 0;          // unique in the process (amk_plan_create numbers plans)
    amk_plan() = default;
    amk_plan(const amk_plan &) = delete;
    amk_plan &operator=(const amk_plan &) = delete;
    ~amk_plan() { delete pos0; }
    // the validator's view
    std::vector<amk_graph_task> gtasks;
    std::vector<amk_graph_wait> gwaits;
    std::vector<int32_t> gsignals;
    std::vector<amk_graph_access> gacc;
    std::vector<amk_graph_buffer> gbufs;
    std::vector<int32_t> gqueue;
    std::vector<int32_t> kind, layer;
    int64_t weight_bytes = 0, kv_row_bytes = 0;
};

// Lowers cfg for n_sms persistent CTAs into *P (no validation).  With pos0,
// the schedule of a step at position 0: no attention level, the O-projection
// takes each head's output from the V rows directly.
int amk_lower(const amk_config *cfg, const amk_options *opt, int n_sms, amk_plan *P,
              int pos0 = 0);
// The producer's cap on bulk-copy bytes in flight per SM for options o:
// inflight_kb KiB, 64 KiB when 0, no cap when negative.
inline uint32_t amk_inflight_bytes(const amk_options *o)
{
    if (o->inflight_kb < 0)
        return 0xffffffffu;
    return (uint32_t)(o->inflight_kb > 0 ? o->inflight_kb : 64) * 1024u;
}

// Bytes of one copy piece for options o: copy_piece_kb KiB, 64 KiB when 0.
inline uint32_t amk_piece_bytes(const amk_options *o)
{
    return (uint32_t)(o->copy_piece_kb > 0 ? o->copy_piece_kb : 64) * 1024u;
}

// A non-owning amk_graph view of P's graph arrays.
void amk_plan_view(const amk_plan *P, amk_graph *g);
// Tensor maps of the Wdown of layers [l0, l0 + n) for a fused FFN (128 bytes
// each, to be copied to 64-byte aligned device memory): a 2-D [hidden][ffn]
// view with boxes of 16 bytes x ffn_box_rows rows.  Returns an amk status.
int amk_encode_down_maps(const amk_plan *P, const amk_weights *w, int l0, int n, void *out);

// Copies plan task t into *out with its device pointers resolved: weight
// rows, row scales and norm gain from w, KV-cache blocks from kv (bf16
// [L][2][nkv][max_ctx][hd]), and its ring geometry (amk_task_geometry).
// packed_down: the handle keeps a packed copy of every Wdown (fused FFN
// slices then stream contiguous column groups; else 2-D tensor-map boxes).
// Host only; reads only host memory.
void amk_resolve_task(const amk_plan *P, const amk_weights *w, const uint16_t *kv, int t,
                      amk::TaskDesc *out, int packed_down);
// The ring geometry of GEMV task d of plan P (the chunk stream its producer
// issues and the warp layout of its consumers); attention tasks get zeros.
void amk_task_geometry(const amk_plan *P, amk::TaskDesc *d, int packed_down);

#endif
