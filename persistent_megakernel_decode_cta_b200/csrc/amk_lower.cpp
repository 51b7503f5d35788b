// amk_lower.cpp -- lowering a Llama-family decoder shape to the per-SM task
// DAG of one decode step, plus the graph the static validator checks.
//
// paperfeed "RightNow-AI/AutoMegaKernel", "How it works", layer 2: model ->
// graph IR -> tiled task DAG -> instruction stream; the schedule knobs are
// tiling, SM assignment and pipelining depth ("RightNow-AI/AutoMegaKernel"
// README, "Two autoresearch loops").  The lowering is deterministic: the same
// shape and knobs always give the same DAG.
//
// Levels of one layer (each a set of independent tasks; a level waits for the
// full count of the previous level's counter):
//   QKV    row tiles of Wq, Wk, Wv; RMSNorm prologue
//   ATTN   (KV head, position chunk) split-K tiles; RoPE, KV append, partials
//   OPROJ  row tiles of Wo; split-K combine prologue, residual epilogue
//   GATEUP row tiles of Wgate/Wup; RMSNorm prologue, SwiGLU epilogue
//   DOWN   row tiles of Wdown; residual epilogue
// then LMHEAD row tiles with a final-RMSNorm prologue and an argmax epilogue.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <vector>

#include "amk.h"
#include "amk_internal.h"
#include "amk_plan.h"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

extern "C" int amk_kernel_smem_bytes(int ring_stages, int stage_bytes, int vec_floats);

namespace {

using amk::TaskDesc;

constexpr int kMaxSmem = 232448;  // 227 KB opt-in shared memory per CTA on sm_100
constexpr int kMaxK = amk::kConsumerThreads * 48;  // activations a lane keeps in registers

int gran_rows(int64_t row_bytes)
{
    int g = 16;
    while (row_bytes % g)
        g >>= 1;
    return 16 / g;  // rows whose bytes are a multiple of 16
}

// Split [0, rows) into about n tiles whose starts are multiples of gran.
std::vector<std::pair<int, int>> tiles(int rows, int n, int gran)
{
    std::vector<std::pair<int, int>> out;
    n = std::max(1, std::min(n, (rows + gran - 1) / gran));
    int prev = 0;
    for (int i = 1; i <= n; ++i) {
        int b = (int)((int64_t)rows * i / n);
        b -= b % gran;
        if (i == n)
            b = rows;
        if (b > prev) {
            out.push_back({prev, b});
            prev = b;
        }
    }
    return out;
}

struct Logical {
    TaskDesc d;
    int64_t cost;  // bytes streamed
};

}  // namespace

int amk_lower(const amk_config *cfg, const amk_options *opt_in, int n_sms, amk_plan *P,
              int pos0)
{
    amk_options opt;
    amk_default_options(&opt);
    if (opt_in) {
        if (opt_in->ring_stages > 0) opt.ring_stages = opt_in->ring_stages;
        if (opt_in->stage_bytes > 0) opt.stage_bytes = opt_in->stage_bytes;
        if (opt_in->attn_splits > 0) opt.attn_splits = opt_in->attn_splits;
        if (opt_in->tasks_per_sm > 0) opt.tasks_per_sm = opt_in->tasks_per_sm;
        if (opt_in->wait_timeout_us > 0) opt.wait_timeout_us = opt_in->wait_timeout_us;
        opt.debug_skip_signal_task = opt_in->debug_skip_signal_task;
        opt.profile = opt_in->profile;
        if (opt_in->l2_prefetch_kb > 0) opt.l2_prefetch_kb = opt_in->l2_prefetch_kb;
        if (opt_in->ffn_fused != 0) opt.ffn_fused = opt_in->ffn_fused;
        if (opt_in->pos0_plan != 0) opt.pos0_plan = opt_in->pos0_plan;
        if (opt_in->inflight_kb != 0) opt.inflight_kb = opt_in->inflight_kb;
        if (opt_in->copy_piece_kb > 0) opt.copy_piece_kb = opt_in->copy_piece_kb;
        if (opt_in->sm_rotate > 0) opt.sm_rotate = opt_in->sm_rotate;
        opt.debug_checks = opt_in->debug_checks;
        if (opt_in->flagged_waits != 0) opt.flagged_waits = opt_in->flagged_waits;
        opt.n_sms = opt_in->n_sms;
    }
    const amk_config &c = *cfg;
    const int h = c.hidden, L = c.n_layers, nh = c.n_heads, nkv = c.n_kv_heads;
    const int hd = c.head_dim, F = c.ffn, V = c.vocab;
    if (h <= 0 || L <= 0 || nh <= 0 || nkv <= 0 || hd <= 0 || F <= 0 || V <= 0 ||
        c.max_ctx <= 0 || n_sms <= 0)
        return amk_set_error(AMK_ERR_INVALID_ARG, "lowering: non-positive shape or SM count");
    if (c.quant != AMK_QUANT_BF16 && c.quant != AMK_QUANT_W8A16 && c.quant != AMK_QUANT_W4A16)
        return amk_set_error(AMK_ERR_INVALID_ARG, "lowering: unknown quant mode %d", c.quant);
    if (!(c.rms_eps >= 0.f) || !(c.rope_theta > 0.f))
        return amk_set_error(AMK_ERR_INVALID_ARG, "lowering: bad rms_eps or rope_theta");
    if (nh % nkv)
        return amk_set_error(AMK_ERR_UNSUPPORTED, "n_heads %% n_kv_heads != 0");
    if (hd % 8)
        return amk_set_error(AMK_ERR_UNSUPPORTED, "head_dim must be a multiple of 8 "
                             "(16-byte KV rows for bulk copies)");
    // ring shape left at 0: 48 KiB stages for int8 weights and 64 KiB for
    // bf16, as many as make 192 KiB.  Measured on B200: 4 x 48 KiB takes
    // 2-6 % off the W8A16 decode steps and adds 2-5 % to the bf16 ones,
    // whose GEMV does less work per byte; the depth at a fixed ring size
    // matters far less than the stage size
    if (opt.stage_bytes <= 0)
        opt.stage_bytes = c.quant != AMK_QUANT_BF16 ? 48 * 1024 : 64 * 1024;
    if (opt.ring_stages <= 0)
        opt.ring_stages = std::max(2, std::min(amk::kMaxStages, 192 * 1024 / opt.stage_bytes));
    if (opt.ring_stages < 2 || opt.ring_stages > amk::kMaxStages || opt.stage_bytes < 1024 ||
        opt.stage_bytes % 1024)
        return amk_set_error(AMK_ERR_INVALID_ARG, "ring_stages in [2,%d], stage_bytes a "
                             "multiple of 1024", amk::kMaxStages);
    // in-flight cap left at 0: 64 KiB, or 96 KiB for bf16 models whose layer
    // streams at least 1 MiB per SM (bandwidth-bound levels: measured on
    // B200, Llama-7B bf16 at KV context 2048 runs 1.2 % faster with 96 KiB,
    // while TinyLlama, SmolLM2 and the int8 shapes gain nothing or lose up
    // to 1 %, their levels being bound by latency, not by the stream)
    if (opt.inflight_kb == 0 && c.quant == AMK_QUANT_BF16) {
        const int64_t layer_bytes =
            2 * ((int64_t)h * (nh * hd + 2 * nkv * hd) + (int64_t)nh * hd * h + 3 * (int64_t)h * F);
        if (layer_bytes / n_sms >= (int64_t)1 << 20)
            opt.inflight_kb = 96;
    }
    const int G = nh / nkv;
    // attention lane layout: lph lanes per head, E = hd / lph elements per
    // lane, the G heads of a group side by side, and as many position groups
    // of lph * G lanes as fit a warp.  By default the heads spread over the
    // warp (lph = largest power of two with lph * G <= 32); heads of 128 or
    // more elements take 16 per lane instead, so that a warp scores several
    // positions at once with fewer shuffle steps (measured: faster for
    // Llama-7B shapes, slower for short chunks of 64-element heads)
    int lph = 32;
    while (lph > 1 && (lph * G > 32 || hd % lph))
        lph >>= 1;
    if (hd >= 128 && hd % 16 == 0 && hd / lph < 16)
        lph = hd / 16;
    const int att_e = hd / lph;
    if (h > 16 * 256 || nh * hd > 16 * 256 || F > 3 * 16 * 256 * 4)
        return amk_set_error(AMK_ERR_UNSUPPORTED, "hidden or heads*head_dim above 4096, or ffn "
                             "above 49152 (prologue register blocking)");
    if (G > 32 || lph * G > 32 || hd % lph || att_e > 16 || (att_e & (att_e - 1)))
        return amk_set_error(AMK_ERR_UNSUPPORTED, "attention layout: group %d x head_dim %d "
                             "does not fit one warp", G, hd);
    // bytes per weight: 2 (bf16), 1 (int8), or 0 for packed int4 rows
    const bool q4 = c.quant == AMK_QUANT_W4A16;
    const int esz = c.quant == AMK_QUANT_W8A16 ? 1 : q4 ? 0 : 2;
    const int head_esz = c.tied_embeddings ? 2 : esz;
    auto rowb = [](int K, int e) -> int64_t { return e ? (int64_t)K * e : amk::q4_row_bytes(K); };
    struct Mat { int rows, K, esz; const char *name; };
    const Mat mats[] = {{nh * hd, h, esz, "wq"}, {nkv * hd, h, esz, "wk"},
                        {nkv * hd, h, esz, "wv"}, {h, nh * hd, esz, "wo"},
                        {F, h, esz, "wgate"},     {F, h, esz, "wup"},
                        {h, F, esz, "wdown"},     {V, h, head_esz, "lm_head"}};
    for (const Mat &m : mats) {
        const int64_t rb = rowb(m.K, m.esz);
        if (m.esz == 0 && m.K % 32)
            return amk_set_error(AMK_ERR_UNSUPPORTED, "%s: W4A16 rows need a multiple of 32 "
                                 "inputs (whole 16-byte code vectors), not %d", m.name, m.K);
        if (m.K > kMaxK)
            return amk_set_error(AMK_ERR_UNSUPPORTED, "%s: inner dimension %d > %d", m.name,
                                 m.K, kMaxK);
        if (rb % 4)
            return amk_set_error(AMK_ERR_UNSUPPORTED, "%s: row of %lld bytes is not a "
                                 "multiple of 4", m.name, (long long)rb);
        if (((int64_t)m.rows * rb) % 16)
            return amk_set_error(AMK_ERR_UNSUPPORTED, "%s: %lld bytes is not a multiple of "
                                 "16", m.name, (long long)(m.rows * rb));
        if ((int64_t)gran_rows(rb) * rb > opt.stage_bytes)
            return amk_set_error(AMK_ERR_UNSUPPORTED, "%s: a row of %lld bytes does not fit a "
                                 "%d-byte ring stage", m.name, (long long)rb, opt.stage_bytes);
    }
    if (4 * hd > opt.stage_bytes)
        return amk_set_error(AMK_ERR_UNSUPPORTED, "head_dim too large for the ring stage");

    // split-K chunks per KV head: as many as keep every attention task of a
    // layer on its own SM, at most 8 (the merge of a head's chunks by the last
    // one to finish then takes two L2 round trips)
    int C = opt.attn_splits;
    if (C <= 0)
        C = std::max(1, std::min(n_sms / nkv, 8));
    C = std::min(C, c.max_ctx);
    // the shared vector holds a prologue's output (the normed hidden state or
    // the attention output, padded by 4 floats per 32 for conflict-free
    // loads), a fused FFN slice's activations, or the attention tile's
    // scratch; DOWN tiles read their activations from L2 directly
    auto padded = [](int n) { return n + n / 32 * 4 + 4; };
    // (and, for a fused FFN slice of int8 weights, its activations as int16
    // pairs at byte 1024: at least 320 floats)
    int vec = std::max({padded(h), padded(nh * hd),
                        G * hd + 2 * hd + amk::kConsumerWarps * G * (hd + 2), 320});
    vec = (vec + 3) & ~3;
    int stages = opt.ring_stages;
    while (stages > 2 && amk_kernel_smem_bytes(stages, opt.stage_bytes, vec) > kMaxSmem)
        --stages;
    const int smem = amk_kernel_smem_bytes(stages, opt.stage_bytes, vec);
    if (smem > kMaxSmem)
        return amk_set_error(AMK_ERR_UNSUPPORTED, "shared memory %d bytes > %d", smem, kMaxSmem);

    P->cfg = c;
    P->opt = opt;
    P->opt.ring_stages = stages;
    P->opt.attn_splits = C;
    P->n_sms = n_sms;
    P->group = G;
    P->qkv_rows = nh * hd + 2 * nkv * hd;
    P->vec_floats = vec;
    P->smem_bytes = smem;
    P->att_lph = lph;
    P->att_hpb = 32 / lph;
    P->att_pg = std::max(1, 32 / (lph * G));
    P->att_e = hd / lph;
    // the generic instance takes odd row widths and a bf16 tied head on int8
    // layers; the int4 instance runs a tied bf16 head itself and has no odd
    // rows (K % 32 == 0 above), so int4 never needs it
    P->generic = (c.tied_embeddings && c.quant == AMK_QUANT_W8A16) ? 1 : 0;
    for (const Mat &m : mats)
        if (rowb(m.K, m.esz) % 16)
            P->generic = 1;
    if (q4 && P->generic)
        return amk_set_error(AMK_ERR_UNSUPPORTED, "W4A16: a tied head of %d-byte rows is not "
                             "a multiple of 16 bytes", h * 2);

    // FFN fusion: the columns [a, b) of Wdown come as 2-D TMA boxes of 16
    // bytes x box_rows rows, so the slice starts and the row pitch must be
    // 16-byte multiples and the box rows must divide hidden
    int box_rows = 0;
    for (int br : {256, 128, 64})
        if (!box_rows && h % br == 0)
            box_rows = br;
    // slice width: a multiple of 16 bytes of a Wdown row, about one slice per
    // SM, at most 128 (the gate/up half of the red buffer)
    // (int4 weights keep separate FFN levels: no fused int4 down projection)
    const int fesz = q4 ? 1 : esz;
    const int ffn_gran = 16 / fesz;
    const int ffn_units = F / ffn_gran, n_target = n_sms * std::max(1, opt.tasks_per_sm);
    const int ffn_w = std::min((ffn_units + n_target - 1) / n_target * ffn_gran,
                               amk::kMaxTaskRows / 2 / ffn_gran * ffn_gran);
    const int64_t ffn_fit = box_rows ? (int64_t)opt.stage_bytes /
                                           ((int64_t)ffn_w * fesz * box_rows) * box_rows
                                     : 0;
    // default (ffn_fused = 1): separate FFN levels with flagged waits.  With
    // level counters (flagged_waits = -1) the default fuses when a residual row
    // is at most 1.5 KB: the fused level adds every slice's partial down
    // projection into the same hidden-sized accumulator with 64-bit atomics,
    // whose contention grows with the width; measured on B200 it gained 3% on
    // the SmolLM2 shape (1152 B) but lost 2% on Llama-1B W8A16 (2 KB), 4% on
    // Llama-7B and 10% on TinyLlama.  A fused level needs the counters (its
    // residual is a fixed-point sum, not flagged words), and separate levels
    // with flagged waits measured faster on the SmolLM2 shape too (517 against
    // 527 us at context 0, 721 against 787 at 128).  ffn_fused = 2 fuses
    // whenever the shape allows.
    const bool shape_ok = !q4 && F % ffn_gran == 0 && box_rows > 0 &&
                          ((int64_t)F * fesz) % 16 == 0 && (ffn_fit >= h || ffn_fit >= 256);
    const bool fused = shape_ok && (opt.ffn_fused >= 2 ||
                                    (opt.ffn_fused == 1 && opt.flagged_waits < 0 &&
                                     (int64_t)h * fesz <= 1536));
    P->ffn_fused = fused ? 1 : 0;
    // flagged waits need every input of every task to be a flagged word: with
    // a fused FFN level the residual is a fixed-point sum, so counters stay
    P->flagged = !fused && opt.flagged_waits >= 0 ? 1 : 0;
    P->ffn_box_rows = fused ? box_rows : 0;

    // ---- logical tasks per level ---------------------------------------------
    // unfused: QKV, ATTN, OPROJ, GATEUP, DOWN; fused: QKV, ATTN, OPROJ, FFN;
    // the position-0 schedule has no ATTN level
    P->is_pos0 = pos0 ? 1 : 0;
    const int LV_N = (fused ? 4 : 5) - (pos0 ? 1 : 0);
    auto ctr_of = [&](int layer, int lv) { return layer * LV_N + lv; };
    const int n_ctr = L * LV_N;
    std::vector<std::vector<Logical>> levels;
    auto mk = [](uint8_t kind, int layer, int r0, int r1, uint8_t mat = 0) {
        TaskDesc d{};
        d.kind = kind;
        d.mat = mat;
        d.layer = layer;
        d.wait_ctr = -1;
        d.signal_ctr = -1;
        d.r0 = r0;
        d.r1 = r1;
        return d;
    };
    const int tps = std::max(1, opt.tasks_per_sm);
    auto gemv_level = [&](uint8_t kind, int layer, int rows, int K, int e, int target,
                          int max_rows, uint8_t mat, std::vector<Logical> &out) {
        const int64_t rb = rowb(K, e);
        int n = std::max(target, (rows + max_rows - 1) / max_rows);
        std::vector<std::pair<int, int>> tl;
        for (;; ++n) {  // granule rounding may grow a tile past max_rows
            tl = tiles(rows, n, gran_rows(rb));
            bool fits = true;
            for (auto t : tl)
                fits &= t.second - t.first <= max_rows;
            if (fits)
                break;
        }
        for (auto t : tl)
            out.push_back({mk(kind, layer, t.first, t.second, mat),
                           (int64_t)(t.second - t.first) * rb});
    };
    for (int l = 0; l < L; ++l) {
        // QKV: tiles shared among the three matrices in proportion to rows
        std::vector<Logical> qkv;
        const int rows3[3] = {nh * hd, nkv * hd, nkv * hd};
        const int total = P->qkv_rows;
        const int target = n_sms * tps;
        int given = 0;
        for (int m = 0; m < 3; ++m) {
            int nt = m < 2 ? std::max(1, (int)((int64_t)target * rows3[m] / total))
                           : std::max(1, target - given);
            given += nt;
            gemv_level(amk::TK_QKV, l, rows3[m], h, esz, nt, amk::kMaxTaskRows, (uint8_t)m, qkv);
        }
        levels.push_back(std::move(qkv));
        if (!pos0) {
            std::vector<Logical> att;
            for (int g = 0; g < nkv; ++g)
                for (int ci = 0; ci < C; ++ci)
                    att.push_back({mk(amk::TK_ATTN, l, g, ci), 0});
            levels.push_back(std::move(att));
        }
        std::vector<Logical> o, gu, dn;
        gemv_level(amk::TK_OPROJ, l, h, nh * hd, esz, target, amk::kMaxTaskRows, 0, o);
        if (pos0)
            for (auto &t : o)
                t.d.flags |= amk::TF_POS0;
        levels.push_back(std::move(o));
        if (fused) {
            std::vector<Logical> ffn;
            for (int a = 0; a < F; a += ffn_w) {
                const int b = std::min(a + ffn_w, F);
                ffn.push_back({mk(amk::TK_FFN, l, a, b), (int64_t)(b - a) * h * esz * 3});
            }
            levels.push_back(std::move(ffn));
            continue;
        }
        gemv_level(amk::TK_GATEUP, l, F, h, esz, target, amk::kMaxTaskRows / 2, 0, gu);
        for (auto &t : gu)
            t.cost *= 2;
        levels.push_back(std::move(gu));
        gemv_level(amk::TK_DOWN, l, h, F, esz, target, amk::kMaxTaskRows, 0, dn);
        levels.push_back(std::move(dn));
    }
    {
        std::vector<Logical> lm;
        gemv_level(amk::TK_LMHEAD, L - 1, V, h, head_esz, n_sms * tps, amk::kMaxTaskRows, 0, lm);
        lm[0].d.flags |= amk::TF_RESET_ARGKEY;
        levels.push_back(std::move(lm));
    }
    // waits / signals: level i of layer l signals ctr(l, i); waits on the
    // previous level's counter at full count (QKV of layer l > 0 waits on
    // the last level of layer l-1; LMHEAD on the last level of the last layer)
    std::vector<uint32_t> total(n_ctr, 0);
    for (size_t li = 0; li + 1 < levels.size(); ++li) {
        const int layer = (int)li / LV_N, lv = (int)li % LV_N;
        for (auto &t : levels[li])
            t.d.signal_ctr = ctr_of(layer, lv);
        total[ctr_of(layer, lv)] = (uint32_t)levels[li].size();
    }
    for (size_t li = 1; li < levels.size(); ++li) {
        const int prev = (int)li - 1;
        const int pc = ctr_of(prev / LV_N, prev % LV_N);
        for (auto &t : levels[li]) {
            t.d.wait_ctr = pc;
            t.d.wait_count = total[pc];
            t.d.wait_total = total[pc];
        }
    }

    // ---- SM assignment: per level, heaviest task to the least-loaded SM --------
    // (ties go to the SM with the least streamed so far, then to the first in
    // the level's scan order, which starts at SM (level * sm_rotate) mod n_sms:
    // the SM-assignment knob moves tiles between SMs without unbalancing them)
    std::vector<std::vector<TaskDesc>> queues(n_sms);
    std::vector<int64_t> cum(n_sms, 0);
    int lvi = 0;
    for (auto &lv : levels) {
        std::vector<int> idx(lv.size());
        std::iota(idx.begin(), idx.end(), 0);
        std::stable_sort(idx.begin(), idx.end(),
                         [&](int a, int b) { return lv[a].cost > lv[b].cost; });
        std::vector<int64_t> load(n_sms, 0);
        std::vector<std::vector<int>> mine(n_sms);
        const int start = (int)(((int64_t)lvi++ * std::max(0, opt.sm_rotate)) % n_sms);
        for (int i : idx) {
            int best = start;
            for (int j = 1; j < n_sms; ++j) {
                const int s = (start + j) % n_sms;
                if (load[s] < load[best] || (load[s] == load[best] && cum[s] < cum[best]))
                    best = s;
            }
            load[best] += std::max<int64_t>(lv[i].cost, 1);
            cum[best] += lv[i].cost;
            mine[best].push_back(i);
        }
        for (int s = 0; s < n_sms; ++s) {
            std::sort(mine[s].begin(), mine[s].end());
            for (int i : mine[s])
                queues[s].push_back(lv[i].d);
        }
    }
    P->tasks.clear();
    P->queue_off.assign(n_sms + 1, 0);
    for (int s = 0; s < n_sms; ++s) {
        P->queue_off[s] = (int32_t)P->tasks.size();
        for (auto &d : queues[s])
            P->tasks.push_back(d);
    }
    P->queue_off[n_sms] = (int32_t)P->tasks.size();
    P->n_counters = n_ctr;
    P->n_arrive = L * nkv;

    // ---- the validator's graph ----------------------------------------------
    const int T = (int)P->tasks.size();
    auto B_QKV = [](int l) { return 6 * l + 0; };
    // the attention output of layer l: the ATTN tasks of KV head g accumulate
    // the heads of g (their split-K partials are merged by whichever chunk
    // task of g arrives last, an arrival-counter protocol inside the kernel:
    // a commutative reduction, modelled as ACCUM)
    auto B_ATTN = [](int l) { return 6 * l + 1; };
    auto B_XMID = [](int l) { return 6 * l + 2; };
    auto B_XOUT = [](int l) { return 6 * l + 3; };
    auto B_ACT = [](int l) { return 6 * l + 4; };
    auto B_KVNEW = [](int l) { return 6 * l + 5; };
    const int B_LOGITS = 6 * L, B_KEY = 6 * L + 1, B_KEYNEXT = 6 * L + 2;
    P->gbufs.assign(6 * L + 3, amk_graph_buffer{0, 0, -1});
    for (int l = 0; l < L; ++l) {
        P->gbufs[B_QKV(l)].size = P->qkv_rows;
        P->gbufs[B_ATTN(l)].size = (int64_t)nh * hd;
        P->gbufs[B_XMID(l)].size = h;
        P->gbufs[B_XOUT(l)].size = h;
        P->gbufs[B_ACT(l)].size = F;
        P->gbufs[B_KVNEW(l)].size = (int64_t)nkv * 2 * hd;
    }
    P->gbufs[B_LOGITS] = {V, AMK_BUF_OUTPUT, -1};
    P->gbufs[B_KEY] = {1, AMK_BUF_OUTPUT, B_KEYNEXT};
    P->gbufs[B_KEYNEXT] = {1, 0, -1};
    P->gtasks.assign(T, amk_graph_task{});
    P->gwaits.clear();
    P->gsignals.clear();
    P->gacc.clear();
    P->kind.assign(T, 0);
    P->layer.assign(T, 0);
    auto acc = [&](int buf, int kind, int64_t b, int64_t e) {
        P->gacc.push_back(amk_graph_access{buf, kind, b, e});
    };
    for (int s = 0; s < n_sms; ++s) {
        for (int t = P->queue_off[s]; t < P->queue_off[s + 1]; ++t) {
            const TaskDesc &d = P->tasks[t];
            amk_graph_task &gt = P->gtasks[t];
            gt.sm = s;
            // with flagged waits the kernel touches no level counter: a task's
            // waits are its flagged reads (READ_FLAGGED accesses below)
            gt.wait_begin = (int32_t)P->gwaits.size();
            if (d.wait_ctr >= 0 && !P->flagged)
                P->gwaits.push_back({d.wait_ctr, (int32_t)d.wait_count});
            gt.wait_count = (int32_t)P->gwaits.size() - gt.wait_begin;
            gt.signal_begin = (int32_t)P->gsignals.size();
            if (d.signal_ctr >= 0 && !P->flagged)
                P->gsignals.push_back(d.signal_ctr);
            gt.signal_count = (int32_t)P->gsignals.size() - gt.signal_begin;
            gt.access_begin = (int32_t)P->gacc.size();
            const int l = d.layer;
            // reads of the activations one level hands to the next
            const int RD = P->flagged ? AMK_ACC_READ_FLAGGED : AMK_ACC_READ;
            // what the kernel's task of this kind reads and writes
            switch (d.kind) {
            case amk::TK_QKV: {
                const int off = d.mat == 0 ? 0 : d.mat == 1 ? nh * hd : (nh + nkv) * hd;
                if (l > 0)
                    acc(B_XOUT(l - 1), RD, 0, h);
                else
                    acc(B_KEYNEXT, AMK_ACC_READ_PREV, 0, 1);
                acc(B_QKV(l), AMK_ACC_WRITE, off + d.r0, off + d.r1);
                break;
            }
            case amk::TK_ATTN: {
                const int g = d.r0, ci = d.r1;
                acc(B_QKV(l), RD, (int64_t)g * G * hd, (int64_t)(g + 1) * G * hd);
                acc(B_QKV(l), RD, (int64_t)nh * hd + g * hd, (int64_t)nh * hd + (g + 1) * hd);
                acc(B_QKV(l), RD, (int64_t)(nh + nkv) * hd + g * hd,
                    (int64_t)(nh + nkv) * hd + (g + 1) * hd);
                acc(B_ATTN(l), AMK_ACC_ACCUM, (int64_t)g * G * hd, (int64_t)(g + 1) * G * hd);
                if (ci == 0)
                    acc(B_KVNEW(l), AMK_ACC_WRITE, (int64_t)g * 2 * hd, (int64_t)(g + 1) * 2 * hd);
                break;
            }
            case amk::TK_OPROJ:
                if (d.flags & amk::TF_POS0) {
                    // head outputs from the V rows; KV row 0 in shares: the tile
                    // of rows [r0, r1) writes (K | V) elements [r0 E / h, r1 E / h)
                    const int64_t E = (int64_t)2 * nkv * hd;
                    acc(B_QKV(l), RD, (int64_t)nh * hd, (int64_t)(nh + 2 * nkv) * hd);
                    if (d.r0 * E / h < d.r1 * E / h)
                        acc(B_KVNEW(l), AMK_ACC_WRITE, d.r0 * E / h, d.r1 * E / h);
                } else {
                    acc(B_ATTN(l), RD, 0, (int64_t)nh * hd);
                }
                if (l > 0)
                    acc(B_XOUT(l - 1), RD, d.r0, d.r1);
                else
                    acc(B_KEYNEXT, AMK_ACC_READ_PREV, 0, 1);
                acc(B_XMID(l), AMK_ACC_WRITE, d.r0, d.r1);
                if (fused)  // the FFN's accumulator starts at the residual
                    acc(B_XOUT(l), AMK_ACC_WRITE, d.r0, d.r1);
                break;
            case amk::TK_FFN:
                acc(B_XMID(l), RD, 0, h);
                acc(B_XOUT(l), AMK_ACC_ACCUM, 0, h);
                break;
            case amk::TK_GATEUP:
                acc(B_XMID(l), RD, 0, h);
                acc(B_ACT(l), AMK_ACC_WRITE, d.r0, d.r1);
                break;
            case amk::TK_DOWN:
                acc(B_ACT(l), RD, 0, F);
                acc(B_XMID(l), RD, d.r0, d.r1);
                acc(B_XOUT(l), AMK_ACC_WRITE, d.r0, d.r1);
                break;
            case amk::TK_LMHEAD:
                acc(B_XOUT(L - 1), RD, 0, h);
                acc(B_LOGITS, AMK_ACC_WRITE, d.r0, d.r1);
                acc(B_KEY, AMK_ACC_ACCUM, 0, 1);
                if (d.flags & amk::TF_RESET_ARGKEY)
                    acc(B_KEYNEXT, AMK_ACC_RESET, 0, 1);
                break;
            }
            gt.access_count = (int32_t)P->gacc.size() - gt.access_begin;
            P->kind[t] = d.kind;
            P->layer[t] = d.layer;
        }
    }
    P->gqueue.resize(T);
    std::iota(P->gqueue.begin(), P->gqueue.end(), 0);

    // ---- bytes streamed per step -------------------------------------------
    int64_t wb = 0;
    for (const Mat &m : mats) {
        const int64_t bytes = (int64_t)m.rows * rowb(m.K, m.esz);  // int4: scales included
        const bool is_head = !strcmp(m.name, "lm_head");
        wb += is_head ? bytes : bytes * L;
        if (m.esz == 1)
            wb += (int64_t)m.rows * 2 * (is_head ? 1 : L);
    }
    wb += (int64_t)(2 * L + 1) * h * 2 + (int64_t)h * 2;  // norm gains + embedding row
    P->weight_bytes = wb;
    P->kv_row_bytes = (int64_t)L * 2 * nkv * hd * 2;
    return AMK_OK;
}

void amk_plan_view(const amk_plan *P, amk_graph *g)
{
    memset(g, 0, sizeof *g);
    g->n_tasks = (int32_t)P->tasks.size();
    g->n_counters = P->n_counters;
    g->n_buffers = (int32_t)P->gbufs.size();
    g->n_sms = P->n_sms;
    g->n_waits = (int32_t)P->gwaits.size();
    g->n_signals = (int32_t)P->gsignals.size();
    g->n_accesses = (int32_t)P->gacc.size();
    g->tasks = P->gtasks.data();
    g->waits = P->gwaits.data();
    g->signals = P->gsignals.data();
    g->accesses = P->gacc.data();
    g->buffers = P->gbufs.data();
    g->queue_offsets = P->queue_off.data();
    g->queue_tasks = P->gqueue.data();
}

void amk_task_geometry(const amk_plan *P, amk::TaskDesc *dp, int packed_down)
{
    amk::TaskDesc &d = *dp;
    d.nchunks = d.ngu = d.rpc = d.nck = d.rpc2 = d.nck2 = d.ncb = 0;
    d.ks_log2 = d.rg_log2 = 0;
    if (d.kind == amk::TK_ATTN)
        return;
    const amk_config &c = P->cfg;
    const int stage = P->opt.stage_bytes;
    constexpr int W = amk::kConsumerWarps;
    // bytes per weight: 2 (bf16), 1 (int8), 0 (packed int4 rows with their scales)
    int K = c.hidden, parts = 1;
    int esz = c.quant == AMK_QUANT_W8A16 ? 1 : c.quant == AMK_QUANT_W4A16 ? 0 : 2;
    if (d.kind == amk::TK_OPROJ)
        K = c.n_heads * c.head_dim;
    else if (d.kind == amk::TK_DOWN)
        K = c.ffn;
    else if (d.kind == amk::TK_GATEUP || d.kind == amk::TK_FFN)
        parts = 2;
    else if (d.kind == amk::TK_LMHEAD && c.tied_embeddings)
        esz = 2;
    const int RB = esz ? K * esz : amk::q4_row_bytes(K), R = d.r1 - d.r0;
    const int gran = gran_rows(RB);
    int rpc = stage / RB;
    rpc -= rpc % gran;
    // warp layout: each lane keeps at most 64 activations of its K-slice in
    // registers.  K is split across more warps when a row needs it, and also
    // while that gives every warp fewer than four rows of a chunk (the GEMV
    // takes rows four at a time) and still leaves each lane a whole vector.
    // int4 rows: 32 codes per 16-byte vector (the scales after them are not
    // vectors of the slice), at most two vectors per lane
    const int VB = (RB % 16 == 0) ? 16 : ((RB % 8 == 0) ? 8 : 4);
    const int NV = esz ? RB / VB : K / 32;
    const int max_vec = esz ? 64 / (VB / esz) : 2;
    const int rows = std::min(rpc, R);
    int KS = 1, ks_log2 = 0;
    while (KS < W) {
        const int rgk = W / KS;
        const bool must = NV > KS * 32 * max_vec || rgk > rpc;
        const bool more_rows = rgk * 4 > rows && NV >= 2 * KS * 32;
        if (!must && !more_rows)
            break;
        KS *= 2;
        ++ks_log2;
    }
    const int RG = W / KS;
    const int step = std::max(RG, gran);  // rows per chunk: a multiple of both
    if (rpc >= step)
        rpc -= rpc % step;
    const int nck = (R + rpc - 1) / rpc;
    int nchunks = nck * parts;
    d.ngu = (uint16_t)nchunks;
    if (d.kind == amk::TK_FFN) {
        const int row_bytes = R * esz, br = P->ffn_box_rows;
        int rpc2;
        if (packed_down) {  // contiguous column groups: any row count per chunk
            rpc2 = std::min(c.hidden, stage / row_bytes);
        } else {            // TMA boxes of br rows
            const int fit = (stage / (row_bytes * br)) * br;  // rows per stage
            rpc2 = fit >= c.hidden ? c.hidden : fit / 256 * 256;
        }
        d.ncb = (uint16_t)(row_bytes / 16);
        d.rpc2 = (uint16_t)rpc2;
        d.nck2 = (uint16_t)((c.hidden + rpc2 - 1) / rpc2);
        nchunks += d.nck2;
    }
    d.nchunks = (uint16_t)nchunks;
    d.rpc = (uint16_t)rpc;
    d.nck = (uint16_t)nck;
    d.ks_log2 = (uint8_t)ks_log2;
    d.rg_log2 = (uint8_t)(3 - ks_log2);
    static_assert(amk::kConsumerWarps == 8, "the row-group log assumes 8 consumer warps");
}

void amk_resolve_task(const amk_plan *P, const amk_weights *w, const uint16_t *kv, int t,
                      amk::TaskDesc *out, int packed_down)
{
    const amk_config &c = P->cfg;
    amk::TaskDesc d = P->tasks[t];
    const int l = d.layer;
    const bool q8 = c.quant == AMK_QUANT_W8A16;
    const bool q4 = c.quant == AMK_QUANT_W4A16;
    // row bytes of a K-input weight row (int4: the packed row, scales included)
    auto rb = [&](int K) -> int64_t {
        return q4 ? amk::q4_row_bytes(K) : (int64_t)K * (q8 ? 1 : 2);
    };
    auto row = [](const void *base, int64_t r, int64_t row_bytes) {
        return static_cast<const void *>(static_cast<const uint8_t *>(base) + r * row_bytes);
    };
    auto srow = [&](const void *const *arr, int64_t r) -> const uint16_t * {
        return q8 ? static_cast<const uint16_t *>(arr[l]) + r : nullptr;
    };
    d.w0 = d.w1 = nullptr;
    d.s0 = d.s1 = d.s2 = d.gain = nullptr;
    const int h = c.hidden;
    switch (d.kind) {
    case amk::TK_QKV: {
        const void *const *mats[3] = {w->wq, w->wk, w->wv};
        const void *const *scs[3] = {w->sq, w->sk, w->sv};
        d.w0 = row(mats[d.mat][l], d.r0, rb(h));
        d.s0 = srow(scs[d.mat], d.r0);
        d.gain = static_cast<const uint16_t *>(w->attn_norm[l]);
        break;
    }
    case amk::TK_ATTN: {
        const size_t blk = (size_t)c.max_ctx * c.head_dim;
        d.w0 = kv + (((size_t)l * 2 + 0) * c.n_kv_heads + d.r0) * blk;
        d.w1 = kv + (((size_t)l * 2 + 1) * c.n_kv_heads + d.r0) * blk;
        break;
    }
    case amk::TK_OPROJ:
        d.w0 = row(w->wo[l], d.r0, rb(c.n_heads * c.head_dim));
        d.s0 = srow(w->so, d.r0);
        break;
    case amk::TK_GATEUP:
        d.w0 = row(w->wgate[l], d.r0, rb(h));
        d.w1 = row(w->wup[l], d.r0, rb(h));
        d.s0 = srow(w->sgate, d.r0);
        d.s1 = srow(w->sup, d.r0);
        d.gain = static_cast<const uint16_t *>(w->ffn_norm[l]);
        break;
    case amk::TK_DOWN:
        d.w0 = row(w->wdown[l], d.r0, rb(c.ffn));
        d.s0 = srow(w->sdown, d.r0);
        break;
    case amk::TK_FFN:  // Wdown comes through the layer's tensor map
        d.w0 = row(w->wgate[l], d.r0, rb(h));
        d.w1 = row(w->wup[l], d.r0, rb(h));
        d.s0 = srow(w->sgate, d.r0);
        d.s1 = srow(w->sup, d.r0);
        d.s2 = srow(w->sdown, 0);
        d.gain = static_cast<const uint16_t *>(w->ffn_norm[l]);
        break;
    default: {  // TK_LMHEAD
        const bool head_q8 = q8 && !c.tied_embeddings;
        d.w0 = row(c.tied_embeddings ? w->embed : w->lm_head, d.r0,
                   c.tied_embeddings ? (int64_t)h * 2 : rb(h));
        d.s0 = head_q8 ? static_cast<const uint16_t *>(w->lm_head_scale) + d.r0 : nullptr;
        d.gain = static_cast<const uint16_t *>(w->final_norm);
        break;
    }
    }
    amk_task_geometry(P, &d, packed_down);
    *out = d;
}

int amk_encode_down_maps(const amk_plan *P, const amk_weights *w, int l0, int n, void *out)
{
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return amk_set_error(AMK_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    const amk_config &c = P->cfg;
    const bool q8 = c.quant == AMK_QUANT_W8A16;
    const int esz = q8 ? 1 : 2;
    for (int l = l0; l < l0 + n; ++l) {
        CUtensorMap map;
        CUtensorMap *m = &map;
        const cuuint64_t dims[2] = {(cuuint64_t)c.ffn, (cuuint64_t)c.hidden};
        const cuuint64_t strides[1] = {(cuuint64_t)c.ffn * esz};
        const cuuint32_t box[2] = {(cuuint32_t)(16 / esz), (cuuint32_t)P->ffn_box_rows};
        const cuuint32_t estr[2] = {1, 1};
        const CUresult r = encode(m, q8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16,
                                  2, const_cast<void *>(w->wdown[l]), dims, strides, box, estr,
                                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS)
            return amk_set_error(AMK_ERR_INVALID_ARG, "layer %d: Wdown tensor map (error %d)", l,
                                 (int)r);
        static_assert(sizeof(CUtensorMap) == 128, "CUtensorMap is 128 bytes");
        memcpy(static_cast<uint8_t *>(out) + 128 * (size_t)(l - l0), &map, sizeof map);
    }
    return AMK_OK;
}
