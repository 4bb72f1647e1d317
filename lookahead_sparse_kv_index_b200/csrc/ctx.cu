// Decode context and the tau cadence ("FlashMemory-DeepSeek-V4 ...
// Lookahead Sparse Attention", gist.science technical summary, section 2.1:
// Periodic Triggering every tau = 64 steps; Scoring Mechanism; Dynamic
// Fetching of every entry with I >= 0.5 from the CPU cold pool; Tiered
// Selection of a fine-grained top-k inside the fetched subset for the core
// attention).
//
// Refresh step (t % tau == 0):  score (full scan) -> select -> [side stream:
// fetch the newly kept rows cold pool -> HBM (fetch.cu; or every kept row with
// full_fetch)] -> top-k over the scan's scores -> wait for the fetch ->
// attention over the hot buffer.
// Other steps: listed re-score of the kept set with the step's indexer query
// -> top-k -> attention.  The host never waits inside a step.
//
// Lookahead (lsa_params.lookahead = L >= 1): window r >= 1's kept set is
// predicted at step r tau - L with that step's indexer query -- after that
// step's own work, a full scan and the selection into a second kept-set buffer
// -- and fetched on the side stream (the cache never evicting a slot the
// current set uses) while steps r tau - L .. r tau - 1 still attend window
// r - 1's set; at step r tau the new set becomes current and the step re-ranks
// it with its own query.  The side-stream work is enqueued outside the step
// graphs (a captured fork must rejoin inside its graph).
//
// Options.  Several indexer layers (section 2.4 "Optimal Configuration"): each
// scan runs once per layer with that layer's keys and (q, w), and the union
// score max_l z_l (union.cu) feeds select and the top-k.  Merged attention set
// (section 2.1 "Architectural Design", HCA chunks retained; section 1, the
// recent tokens): the window and HCA rows live after the hot buffer in one KV
// arena, and a row-list merge (attn_set.cu) precedes the attention.
// Host-buffer steps: inputs through two staging slots on a copy stream (a
// call's copies overlap the previous call's kernels); outputs written straight
// into mapped pinned host memory, else staged and copied.
//
// CUDA graphs: after one eager run of each step kind (refresh / listed), a
// step is captured once per distinct set of input and output pointers and
// replayed with one graph launch; a decode loop that reuses its buffers runs
// two graphs.  Stage timing runs the kernels eagerly.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <unordered_map>
#include <vector>

#include "lsa_internal.cuh"

// Step kinds: a refresh (scan, select, fetch, top-k over the scan's scores, attention), a listed step
// (re-score of the current kept set, top-k, attention), and with lookahead a predicting step (a listed step,
// then the scan and selection of the next window's set into the other kept-set buffer).
enum StepKind { kRefresh = 0, kListed = 1, kPredict = 2, kKinds = 3 };

struct GraphKey {
    int kind, set;
    const void *q, *w, *Q;
    void *out;
    float *lse;
    bool operator==(const GraphKey &o) const {
        return kind == o.kind && set == o.set && q == o.q && w == o.w && Q == o.Q && out == o.out && lse == o.lse;
    }
};
struct GraphKeyHash {
    size_t operator()(const GraphKey &k) const {
        size_t h = size_t(k.kind) * 2 + size_t(k.set);
        for (const void *p : {k.q, k.w, k.Q, static_cast<const void *>(k.out), static_cast<const void *>(k.lse)})
            h = h * 1000003u ^ std::hash<const void *>()(p);
        return h;
    }
};
struct GraphEntry {
    cudaGraphExec_t exec;
    int64_t kernels;
};

struct lsa_ctx {
    lsa_params p{};
    std::vector<int64_t> seq_off_h;
    int device = 0;
    int tau = 64;
    float scale = 1.f;
    const void *cold_dev = nullptr;
    int64_t *seq_off_d = nullptr;
    float *z = nullptr;
    float *z_kept = nullptr;
    // kept sets: the current one (cur) and, with lookahead, the next window's, written while cur is in use
    struct KeptSet {
        int32_t *kept_idx = nullptr;
        int64_t *kept_off = nullptr;
        int32_t *kept_slot = nullptr;   // [cap] hot slot of each kept position
        void *kc[lsa::kMaxUnionLayers] = {};    // compacted kept keys per layer (kept-list order)
        float *sc[lsa::kMaxUnionLayers] = {};   // their e4m3 row scales
    } ks[2];
    int cur = 0, n_sets = 1;
    int lookahead = 0;
    bool predicted = false;   // the other set holds a predicted set whose fetch was enqueued
    cudaEvent_t ev_pred = nullptr, ev_pend = nullptr;
    int32_t *slot_of = nullptr;
    void *hot = nullptr;
    int32_t *topk_idx = nullptr, *topk_pos = nullptr, *topk_cnt = nullptr;
    int32_t *err = nullptr;
    // hot-buffer cache (incremental fetch)
    int32_t *owner = nullptr;       // [cap] entry held by each slot, or -1
    int64_t *fetched = nullptr;     // rows fetched by the last refresh
    void *fetch_ws = nullptr;
    cudaEvent_t ev_assign = nullptr;
    // indexer layers (OR-mode union): keys and scales per layer, per-layer scores
    int n_layers = 1;
    const void *k_layer[lsa::kMaxUnionLayers] = {};
    const float *ks_layer[lsa::kMaxUnionLayers] = {};
    float *z_layers = nullptr;    // [n_layers, n_total] full-scan scores (n_layers >= 2)
    float *zk_layers = nullptr;   // [n_layers, kept_capacity] listed scores (n_layers >= 2)
    // compacted kept keys (and e4m3 row scales) per layer, in kept-list order, written at each refresh; the
    // listed re-score streams them with the full tensor-core scan (when the shape runs on the tensor cores)
    bool compact = false;
    int64_t sc_len = 0;
    // merged attention set: window and HCA rows live in the arena after the hot buffer
    bool merged = false;
    int64_t win_base = 0, hca_base = 0, row_cap = 0;
    int64_t *hca_off_d = nullptr;
    int32_t *attn_rows = nullptr;
    void *sel_ws = nullptr;
    size_t sel_ws_bytes = 0;
    void *attn_ws = nullptr;
    size_t attn_ws_bytes = 0;
    // staging for lsa_decode_step_host: two slots, so that the inputs of one
    // step cross the host link while the previous step's kernels run
    struct Staging {
        void *q = nullptr, *Q = nullptr, *out = nullptr;
        float *w = nullptr, *lse = nullptr;
        cudaEvent_t in_ready = nullptr;   // the slot's inputs have landed (copy stream)
        cudaEvent_t used = nullptr;       // the slot's step has run (caller's stream)
        cudaEvent_t lse_done = nullptr;   // the slot's lse has reached the host
    } stage[2];
    int64_t host_calls = 0;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaStream_t side = nullptr;
    cudaEvent_t ev_sel = nullptr, ev_gather = nullptr;
    bool refreshed = false;
    // timing
    bool timing = false;
    struct Pending { int stage; cudaEvent_t a, b; };
    std::vector<Pending> pending;
    std::vector<cudaEvent_t> free_events;
    double ms[LSA_STAGE_COUNT] = {0};
    int64_t calls[LSA_STAGE_COUNT] = {0};
    int64_t launches = 0;
    // graphs
    bool use_graphs = true;
    bool eager_done[kKinds * 2] = {};
    cudaStream_t cap = nullptr;
    std::unordered_map<GraphKey, GraphEntry, GraphKeyHash> graphs;
};

namespace {

using namespace lsa;

void free_all(lsa_ctx *c) {
    void *bufs[] = {c->seq_off_d, c->z, c->z_kept, c->slot_of, c->hot,
                    c->topk_idx, c->topk_pos, c->topk_cnt, c->err, c->sel_ws, c->attn_ws,
                    c->owner, c->fetched, c->fetch_ws, c->hca_off_d, c->attn_rows, c->z_layers,
                    c->zk_layers};
    for (void *b : bufs)
        if (b) cudaFree(b);
    for (auto &k : c->ks) {
        for (void *b : {static_cast<void *>(k.kept_idx), static_cast<void *>(k.kept_off),
                        static_cast<void *>(k.kept_slot)})
            if (b) cudaFree(b);
        for (int l = 0; l < lsa::kMaxUnionLayers; ++l) {
            if (k.kc[l]) cudaFree(k.kc[l]);
            if (k.sc[l]) cudaFree(k.sc[l]);
        }
    }
    if (c->ev_pred) cudaEventDestroy(c->ev_pred);
    if (c->ev_pend) cudaEventDestroy(c->ev_pend);
    for (auto &sg : c->stage) {
        for (void *b : {sg.q, sg.Q, sg.out, static_cast<void *>(sg.w), static_cast<void *>(sg.lse)})
            if (b) cudaFree(b);
        for (cudaEvent_t e : {sg.in_ready, sg.used, sg.lse_done})
            if (e) cudaEventDestroy(e);
    }
    if (c->h2d) cudaStreamDestroy(c->h2d);
    if (c->d2h) cudaStreamDestroy(c->d2h);
    if (c->ev_sel) cudaEventDestroy(c->ev_sel);
    if (c->ev_gather) cudaEventDestroy(c->ev_gather);
    if (c->ev_assign) cudaEventDestroy(c->ev_assign);
    for (auto &pe : c->pending) { cudaEventDestroy(pe.a); cudaEventDestroy(pe.b); }
    for (auto e : c->free_events) cudaEventDestroy(e);
    for (auto &g : c->graphs) cudaGraphExecDestroy(g.second.exec);
    c->graphs.clear();
    if (c->side) cudaStreamDestroy(c->side);
    if (c->cap) cudaStreamDestroy(c->cap);
}

constexpr size_t kMaxGraphs = 256;
constexpr int kPredictFetchCtas = 32;

// The device address of page-locked host memory mapped for the device, else nullptr.
void *mapped_host(const void *p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}

cudaEvent_t take_event(lsa_ctx *c) {
    if (!c->free_events.empty()) {
        cudaEvent_t e = c->free_events.back();
        c->free_events.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Brackets one stage with events when timing is on.
struct StageTimer {
    lsa_ctx *c;
    int stage;
    cudaStream_t st;
    cudaEvent_t a = nullptr;
    StageTimer(lsa_ctx *c_, int stage_, cudaStream_t st_) : c(c_), stage(stage_), st(st_) {
        if (c->timing) {
            a = take_event(c);
            cudaEventRecord(a, st);
        }
    }
    void done() {
        if (a) {
            cudaEvent_t b = take_event(c);
            cudaEventRecord(b, st);
            c->pending.push_back({stage, a, b});
            a = nullptr;
        }
    }
};

#define LSA_TRY(call)                       \
    do {                                    \
        lsa_status s_ = (call);             \
        if (s_ != LSA_OK) return s_;        \
    } while (0)

template <typename T>
lsa_status alloc(T **p, size_t bytes) {
    *p = nullptr;
    if (bytes == 0) bytes = 16;
    LSA_CUDA(cudaMalloc(reinterpret_cast<void **>(p), bytes));
    return LSA_OK;
}

// Full scan(s) of every entry with (q, w), the layers' union, and the selection into kept set `set`.
lsa_status enqueue_scan_select(lsa_ctx *c, const void *q, const float *w, int set, cudaStream_t st) {
    const lsa_params &p = c->p;
    const size_t q_layer = size_t(p.B) * p.H * p.d * elem_size(p.q_dtype);   // bytes of one layer's q
    const size_t w_layer = size_t(p.B) * p.H;                                 // floats of one layer's w
    StageTimer ts(c, LSA_STAGE_SCORE, st);
    if (c->n_layers == 1) {
        // one indexer layer: the scan with the selection fused into it (the select stage is then empty)
        LSA_TRY(launch_index_score_select(q, p.q_dtype, w, p.k_dev, p.k_dtype, p.k_scale_dev, c->seq_off_d,
                                          p.n_total, p.B, p.H, p.d, c->z, c->ks[set].kept_idx, p.kept_capacity,
                                          c->ks[set].kept_off, c->sel_ws, c->err, st));
        ts.done();
        StageTimer tsel(c, LSA_STAGE_SELECT, st);
        tsel.done();
        return LSA_OK;
    } else {
        const float *zl[kMaxUnionLayers];
        for (int l = 0; l < c->n_layers; ++l) {
            float *z_l = c->z_layers + size_t(l) * p.n_total;
            LSA_TRY(launch_index_score(static_cast<const char *>(q) + l * q_layer, p.q_dtype, w + l * w_layer,
                                       c->k_layer[l], p.k_dtype, c->ks_layer[l], c->seq_off_d, p.n_total, nullptr,
                                       nullptr, 0, p.B, p.H, p.d, z_l, nullptr, 0, c->err, st));
            zl[l] = z_l;
        }
        LSA_TRY(launch_union(zl, c->n_layers, p.n_total, c->z, st));
    }
    ts.done();
    StageTimer tsel(c, LSA_STAGE_SELECT, st);
    LSA_TRY(launch_select(c->z, c->seq_off_d, p.n_total, p.B, c->ks[set].kept_idx, p.kept_capacity,
                          c->ks[set].kept_off, nullptr, c->sel_ws, c->err, st));
    tsel.done();
    return LSA_OK;
}

// The cold-pool fetch of kept set `set` (the cache never evicting the slots of kept set `protect`, or none
// when protect < 0), then the compaction of its keys; on the side stream.
lsa_status enqueue_fetch(lsa_ctx *c, int set, int protect, cudaStream_t side) {
    const lsa_params &p = c->p;
    const int64_t cap = p.kept_capacity;
    auto &k = c->ks[set];
    StageTimer tg(c, LSA_STAGE_GATHER, side);
    if (p.full_fetch) {
        LSA_TRY(launch_gather(c->cold_dev, p.row_bytes, c->seq_off_d, p.n_total, k.kept_idx, k.kept_off, p.B, c->hot,
                              cap, c->slot_of, c->err, side));
    } else {
        LSA_TRY(launch_fetch(c->cold_dev, p.row_bytes, c->seq_off_d, k.kept_idx, k.kept_off, p.B, c->hot, cap,
                             c->slot_of, c->owner, k.kept_slot, c->fetched, c->fetch_ws, c->err, c->ev_assign, side,
                             protect >= 0 ? c->ks[protect].kept_slot : nullptr,
                             protect >= 0 ? c->ks[protect].kept_off : nullptr,
                             // under running decode steps the host-link copy takes few SMs (32 CTAs keep ~1 MB of
                             // zero-copy reads in flight, far more than the link's bandwidth-delay product)
                             protect >= 0 ? kPredictFetchCtas : 0));
    }
    if (c->compact)
        for (int l = 0; l < c->n_layers; ++l)
            LSA_TRY(launch_gather_keys(c->k_layer[l], int64_t(p.d) * int64_t(elem_size(p.k_dtype)), c->ks_layer[l],
                                       c->seq_off_d, k.kept_idx, k.kept_off, p.B, cap, k.kc[l], k.sc[l], side));
    tg.done();
    return LSA_OK;
}

// Re-score of kept set `set` with this step's (q, w), the layers' union, then the top-k.
lsa_status enqueue_rescore_topk(lsa_ctx *c, const void *q, const float *w, int set, cudaStream_t st) {
    const lsa_params &p = c->p;
    const int64_t cap = p.kept_capacity;
    const size_t q_layer = size_t(p.B) * p.H * p.d * elem_size(p.q_dtype);
    const size_t w_layer = size_t(p.B) * p.H;
    auto &k = c->ks[set];
    StageTimer tr(c, LSA_STAGE_RESCORE, st);
    const bool compact = c->compact && aligned16(q);   // the tensor-core scan reads q with 16-byte loads
    if (compact) {
        // the kept keys in kept-list order: z lands at the kept position
        const float *zl[kMaxUnionLayers];
        for (int l = 0; l < c->n_layers; ++l) {
            float *z_l = c->n_layers == 1 ? c->z_kept : c->zk_layers + size_t(l) * cap;
            LSA_TRY(launch_index_score_tc_axis(static_cast<const char *>(q) + l * q_layer, w + l * w_layer, k.kc[l],
                                               p.k_dtype, k.sc[l], c->sc_len, k.kept_off, cap, cap, p.B, p.H, p.d,
                                               z_l, c->err, st));
            zl[l] = z_l;
        }
        if (c->n_layers > 1) LSA_TRY(launch_union(zl, c->n_layers, cap, c->z_kept, st));
    } else if (c->n_layers == 1) {
        LSA_TRY(launch_index_score(q, p.q_dtype, w, p.k_dev, p.k_dtype, p.k_scale_dev, c->seq_off_d, p.n_total,
                                   k.kept_idx, k.kept_off, cap, p.B, p.H, p.d, c->z_kept, nullptr, 0, c->err, st));
    } else {
        // every layer re-scores the kept set; the ranking score is their union (positions past the
        // kept total hold stale values that the top-k never reads)
        const float *zl[kMaxUnionLayers];
        for (int l = 0; l < c->n_layers; ++l) {
            float *z_l = c->zk_layers + size_t(l) * cap;
            LSA_TRY(launch_index_score(static_cast<const char *>(q) + l * q_layer, p.q_dtype, w + l * w_layer,
                                       c->k_layer[l], p.k_dtype, c->ks_layer[l], c->seq_off_d, p.n_total,
                                       k.kept_idx, k.kept_off, cap, p.B, p.H, p.d, z_l, nullptr, 0, c->err, st));
            zl[l] = z_l;
        }
        LSA_TRY(launch_union(zl, c->n_layers, cap, c->z_kept, st));
    }
    tr.done();
    StageTimer tk(c, LSA_STAGE_TOPK, st);
    LSA_TRY(launch_topk(c->z_kept, 0, c->seq_off_d, k.kept_idx, k.kept_off, p.B, p.topk, cap,
                        p.full_fetch ? nullptr : k.kept_slot, c->topk_idx, c->topk_pos, c->topk_cnt, st));
    tk.done();
    return LSA_OK;
}

lsa_status enqueue_attention(lsa_ctx *c, const void *Q, void *out, float *lse, cudaStream_t st) {
    const lsa_params &p = c->p;
    StageTimer ta(c, LSA_STAGE_ATTN, st);
    if (c->merged) {
        LSA_TRY(launch_merge_rows(c->topk_idx, c->topk_pos, c->topk_cnt, c->seq_off_d, p.B, p.topk, p.window,
                                  int32_t(c->win_base), c->hca_off_d, int32_t(c->hca_base), c->attn_rows,
                                  int32_t(c->row_cap), nullptr, c->err, st));
        LSA_TRY(launch_sparse_attn(Q, p.attn_dtype, c->hot, p.kv_row_stride, p.k_off, p.v_off, c->attn_rows, p.B,
                                   p.Hq, p.D, int32_t(c->row_cap), c->scale, out, lse, c->attn_ws, c->err, st));
    } else {
        LSA_TRY(launch_sparse_attn(Q, p.attn_dtype, c->hot, p.kv_row_stride, p.k_off, p.v_off, c->topk_pos, p.B,
                                   p.Hq, p.D, p.topk, c->scale, out, lse, c->attn_ws, c->err, st));
    }
    ta.done();
    return LSA_OK;
}

// The kernels of one step of kind `kind` on kept set `set` (a predicting step also scans and selects into
// the other set; its fetch is enqueued by run_step, outside any graph).
lsa_status enqueue_step(lsa_ctx *c, int kind, int set, const void *q, const float *w, const void *Q, void *out,
                        float *lse, cudaStream_t st) {
    const lsa_params &p = c->p;
    if (kind == kRefresh) {
        LSA_TRY(enqueue_scan_select(c, q, w, set, st));
        LSA_CUDA(cudaEventRecord(c->ev_sel, st));
        LSA_CUDA(cudaStreamWaitEvent(c->side, c->ev_sel, 0));
        LSA_TRY(enqueue_fetch(c, set, -1, c->side));
        LSA_CUDA(cudaEventRecord(c->ev_gather, c->side));
        // the top-k writes hot slots: with the cache it needs the slot assignment first
        if (!p.full_fetch) LSA_CUDA(cudaStreamWaitEvent(st, c->ev_assign, 0));
        StageTimer tk(c, LSA_STAGE_TOPK, st);
        LSA_TRY(launch_topk(c->z, 1, c->seq_off_d, c->ks[set].kept_idx, c->ks[set].kept_off, p.B, p.topk,
                            p.kept_capacity, p.full_fetch ? nullptr : c->ks[set].kept_slot, c->topk_idx, c->topk_pos,
                            c->topk_cnt, st));
        tk.done();
        LSA_CUDA(cudaStreamWaitEvent(st, c->ev_gather, 0));
        return enqueue_attention(c, Q, out, lse, st);
    }
    LSA_TRY(enqueue_rescore_topk(c, q, w, set, st));
    LSA_TRY(enqueue_attention(c, Q, out, lse, st));
    if (kind == kPredict) LSA_TRY(enqueue_scan_select(c, q, w, set ^ 1, st));
    return LSA_OK;
}

lsa_status launch_step(lsa_ctx *c, int kind, int set, const void *q, const float *w, const void *Q, void *out,
                       float *lse, cudaStream_t st) {
    const int slot = kind * 2 + set;
    if (c->use_graphs && !c->timing && c->eager_done[slot]) {
        const GraphKey key{kind, set, q, w, Q, out, lse};
        auto it = c->graphs.find(key);
        if (it == c->graphs.end()) {
            if (c->graphs.size() >= kMaxGraphs) {
                for (auto &g : c->graphs) cudaGraphExecDestroy(g.second.exec);
                c->graphs.clear();
            }
            LSA_CUDA(cudaStreamBeginCapture(c->cap, cudaStreamCaptureModeThreadLocal));
            const int64_t l0 = launch_count();
            const lsa_status s = enqueue_step(c, kind, set, q, w, Q, out, lse, c->cap);
            cudaGraph_t g = nullptr;
            const cudaError_t e = cudaStreamEndCapture(c->cap, &g);
            if (s != LSA_OK || e != cudaSuccess) {
                if (g) cudaGraphDestroy(g);
                cudaGetLastError();
                if (s != LSA_OK) return s;
                set_error("lsa_decode_step: stream capture failed: %s", cudaGetErrorString(e));
                return LSA_ERR_CUDA;
            }
            cudaGraphExec_t exec = nullptr;
            const cudaError_t ie = cudaGraphInstantiate(&exec, g, 0);
            cudaGraphDestroy(g);
            if (ie != cudaSuccess) {
                set_error("lsa_decode_step: graph instantiation failed: %s", cudaGetErrorString(ie));
                return LSA_ERR_CUDA;
            }
            it = c->graphs.emplace(key, GraphEntry{exec, launch_count() - l0}).first;
        }
        LSA_CUDA(cudaGraphLaunch(it->second.exec, st));
        c->launches += it->second.kernels;
    } else {
        const int64_t l0 = launch_count();
        LSA_TRY(enqueue_step(c, kind, set, q, w, Q, out, lse, st));
        c->launches += launch_count() - l0;
        c->eager_done[slot] = true;
    }
    return LSA_OK;
}

lsa_status run_step(lsa_ctx *c, int64_t t, const void *q, const float *w, const void *Q, void *out,
                    float *lse, cudaStream_t st) {
    const int L = c->lookahead;
    int kind;
    if (!c->refreshed) {
        kind = kRefresh;
    } else if (L == 0) {
        kind = (t % c->tau) == 0 ? kRefresh : kListed;
    } else if (t % c->tau == 0) {
        // window start: the predicted set becomes current once its fetch has landed; without a prediction
        // (the caller skipped its step) the window refreshes here
        kind = c->predicted ? kListed : kRefresh;
        if (c->predicted) {
            LSA_CUDA(cudaStreamWaitEvent(st, c->ev_pend, 0));
            c->cur ^= 1;
            c->predicted = false;
        }
    } else {
        kind = (t + L) % c->tau == 0 ? kPredict : kListed;
    }
    const int set = c->cur;
    LSA_TRY(launch_step(c, kind, set, q, w, Q, out, lse, st));
    if (kind == kRefresh) {
        c->refreshed = true;
        c->predicted = false;
    } else if (kind == kPredict) {
        // the next window's fetch and key compaction run on the side stream while this window's
        // remaining steps run; the window's first step waits for them
        LSA_CUDA(cudaEventRecord(c->ev_pred, st));
        LSA_CUDA(cudaStreamWaitEvent(c->side, c->ev_pred, 0));
        const int64_t l0 = launch_count();
        LSA_TRY(enqueue_fetch(c, set ^ 1, set, c->side));
        c->launches += launch_count() - l0;
        LSA_CUDA(cudaEventRecord(c->ev_pend, c->side));
        c->predicted = true;
    }
    return LSA_OK;
}

}  // namespace

extern "C" {

lsa_status lsa_ctx_create(const lsa_params *pp, lsa_ctx **out) {
    clear_error();
    LSA_CHECK_ARG(pp && out, "lsa_ctx_create: params and out are required");
    *out = nullptr;
    const lsa_params &p = *pp;
    LSA_CHECK_ARG(p.B >= 1 && p.H >= 1 && p.d >= 1 && p.Hq >= 1 && p.D >= 1 && p.topk >= 1,
                  "lsa_ctx_create: sizes must be positive");
    LSA_CHECK_ARG(p.n_total >= 0 && p.n_total < (int64_t(1) << 31), "lsa_ctx_create: n_total out of range");
    LSA_CHECK_ARG(p.seq_off_host && p.k_dev && p.cold_host, "lsa_ctx_create: seq_off_host, k_dev, cold_host required");
    LSA_CHECK_ARG(p.tau >= 0, "lsa_ctx_create: tau < 0");
    LSA_CHECK_ARG(p.kept_capacity >= 1, "lsa_ctx_create: kept_capacity must be >= 1");
    LSA_CHECK_ARG(p.row_bytes > 0 && p.row_bytes % 16 == 0, "lsa_ctx_create: row_bytes must be a multiple of 16");
    LSA_CHECK_ARG(p.kv_row_stride * int64_t(elem_size(p.attn_dtype)) == p.row_bytes,
                  "lsa_ctx_create: kv_row_stride * element size must equal row_bytes");
    LSA_CHECK_SUPPORTED(p.attn_dtype == LSA_F32 || p.attn_dtype == LSA_BF16, "lsa_ctx_create: attn dtype");
    LSA_CHECK_SUPPORTED(p.q_dtype == LSA_F32 || p.q_dtype == LSA_BF16, "lsa_ctx_create: q dtype");
    LSA_CHECK_ARG(valid_dtype(p.k_dtype) && ((p.k_dtype == LSA_E4M3) == (p.k_scale_dev != nullptr)),
                  "lsa_ctx_create: k_scale_dev is required for E4M3 keys and only for them");
    LSA_CHECK_SUPPORTED(p.H <= 64 && (p.d == 32 || p.d == 64 || p.d == 128), "lsa_ctx_create: H/d");
    LSA_CHECK_SUPPORTED(p.D % 32 == 0 && p.D <= 512 && p.Hq <= 256 && p.topk <= 4096, "lsa_ctx_create: Hq/D/topk");
    LSA_CHECK_ARG(p.k_off >= 0 && p.v_off >= 0 && p.k_off + p.D <= p.kv_row_stride && p.v_off + p.D <= p.kv_row_stride,
                  "lsa_ctx_create: K/V must lie inside a row");
    const int64_t *so = p.seq_off_host;
    LSA_CHECK_ARG(so[0] == 0 && so[p.B] == p.n_total, "lsa_ctx_create: seq_off must run from 0 to n_total");
    for (int b = 0; b < p.B; ++b)
        LSA_CHECK_ARG(so[b + 1] >= so[b], "lsa_ctx_create: seq_off must be non-decreasing");
    LSA_CHECK_ARG(p.window >= 0, "lsa_ctx_create: window < 0");
    const int tau = p.tau ? p.tau : 64;
    LSA_CHECK_ARG(p.lookahead >= 0 && p.lookahead < tau, "lsa_ctx_create: lookahead=%d must lie in [0, tau)",
                  p.lookahead);
    LSA_CHECK_SUPPORTED(p.lookahead == 0 || !p.full_fetch,
                        "lsa_ctx_create: lookahead needs the cached hot buffer (full_fetch = 0)");
    const int n_layers = p.n_layers <= 1 ? 1 : p.n_layers;
    LSA_CHECK_ARG(n_layers <= kMaxUnionLayers, "lsa_ctx_create: n_layers=%d > %d", p.n_layers, kMaxUnionLayers);
    if (n_layers > 1) {
        LSA_CHECK_ARG(p.k_dev_layers, "lsa_ctx_create: n_layers >= 2 needs k_dev_layers");
        LSA_CHECK_ARG(p.k_dtype != LSA_E4M3 || p.k_scale_layers, "lsa_ctx_create: E4M3 layers need k_scale_layers");
        for (int l = 1; l < n_layers; ++l) {
            LSA_CHECK_ARG(p.k_dev_layers[l - 1], "lsa_ctx_create: layer %d has no keys", l);
            LSA_CHECK_ARG((p.k_dtype == LSA_E4M3) == (p.k_scale_layers && p.k_scale_layers[l - 1] != nullptr),
                          "lsa_ctx_create: layer %d: a row-scale pointer for E4M3 keys and only for them", l);
        }
    }
    LSA_CHECK_ARG(!p.hca_rows || p.hca_off_host, "lsa_ctx_create: hca_rows needs hca_off_host");
    int64_t n_hca = 0, max_hca = 0;
    if (p.hca_rows) {
        const int64_t *ho = p.hca_off_host;
        LSA_CHECK_ARG(ho[0] == 0, "lsa_ctx_create: hca_off_host[0] must be 0");
        for (int b = 0; b < p.B; ++b) {
            LSA_CHECK_ARG(ho[b + 1] >= ho[b], "lsa_ctx_create: hca_off_host must be non-decreasing");
            max_hca = std::max(max_hca, ho[b + 1] - ho[b]);
        }
        n_hca = ho[p.B];
    }
    const bool merged = p.window > 0 || n_hca > 0;
    const int64_t row_cap = merged ? int64_t(p.topk) + p.window + max_hca : p.topk;
    const int64_t arena_rows = p.kept_capacity + (merged ? int64_t(p.B) * p.window + n_hca : 0);
    LSA_CHECK_SUPPORTED(row_cap <= 65536, "lsa_ctx_create: topk + window + HCA rows per sequence > 65536");
    LSA_CHECK_ARG(arena_rows < (int64_t(1) << 31), "lsa_ctx_create: hot buffer, window and HCA rows exceed 2^31");

    cudaPointerAttributes attr;
    cudaError_t e = cudaPointerGetAttributes(&attr, p.cold_host);
    if (e != cudaSuccess) cudaGetLastError();
    LSA_CHECK_ARG(e == cudaSuccess && attr.type == cudaMemoryTypeHost && attr.devicePointer,
                  "lsa_ctx_create: cold_host is not page-locked host memory mapped for the device");

    lsa_ctx *c = new lsa_ctx();
    c->p = p;
    c->seq_off_h.assign(so, so + p.B + 1);
    c->p.seq_off_host = c->seq_off_h.data();
    c->tau = tau;
    c->lookahead = p.lookahead;
    c->n_sets = p.lookahead > 0 ? 2 : 1;
    c->scale = p.scale > 0.f ? p.scale : 1.f / std::sqrt(float(p.D));
    c->cold_dev = attr.devicePointer;
    cudaGetDevice(&c->device);

    const int64_t cap = p.kept_capacity;
    const size_t qbytes = size_t(p.B) * p.H * p.d * elem_size(p.q_dtype);
    const size_t Qbytes = size_t(p.B) * p.Hq * p.D * elem_size(p.attn_dtype);
    c->sel_ws_bytes = index_score_select_workspace(p.n_total, p.B);   // covers lsa_select's layout too
    c->attn_ws_bytes = sparse_attn_workspace(p.B, p.Hq, p.D, int32_t(row_cap));
    c->merged = merged;
    c->n_layers = n_layers;
    c->k_layer[0] = p.k_dev;
    c->ks_layer[0] = p.k_scale_dev;
    for (int l = 1; l < n_layers; ++l) {
        c->k_layer[l] = p.k_dev_layers[l - 1];
        c->ks_layer[l] = p.k_scale_layers ? p.k_scale_layers[l - 1] : nullptr;
    }
    c->p.k_dev_layers = nullptr;     // the caller's arrays are not kept
    c->p.k_scale_layers = nullptr;
    c->p.hca_rows = nullptr;         // copied into the arena below
    c->p.hca_off_host = nullptr;
    c->row_cap = row_cap;
    c->win_base = cap;
    c->hca_base = cap + int64_t(p.B) * p.window;
    lsa_status s = LSA_OK;
#define LSA_ALLOC(ptr, bytes) \
    if (s == LSA_OK) s = alloc(&(ptr), (bytes))
    LSA_ALLOC(c->seq_off_d, size_t(p.B + 1) * 8);
    LSA_ALLOC(c->z, size_t(p.n_total) * 4);
    LSA_ALLOC(c->z_kept, size_t(cap) * 4);
    for (int k = 0; k < c->n_sets; ++k) {
        LSA_ALLOC(c->ks[k].kept_idx, size_t(cap) * 4);
        LSA_ALLOC(c->ks[k].kept_off, size_t(p.B + 1) * 8);
        LSA_ALLOC(c->ks[k].kept_slot, size_t(cap) * 4);
    }
    LSA_ALLOC(c->slot_of, size_t(p.n_total) * 4);
    LSA_ALLOC(c->hot, size_t(arena_rows) * p.row_bytes);
    if (n_layers > 1) {
        LSA_ALLOC(c->z_layers, size_t(n_layers) * p.n_total * 4);
        LSA_ALLOC(c->zk_layers, size_t(n_layers) * cap * 4);
    }
    if (merged) {
        LSA_ALLOC(c->hca_off_d, size_t(p.B + 1) * 8);
        LSA_ALLOC(c->attn_rows, size_t(p.B) * row_cap * 4);
    }
    // the compacted kept keys, when the listed re-score runs on the tensor cores
    c->compact = index_score_tc_supported(p.q_dtype, p.k_dtype, cap, p.B, p.H, p.d);
    c->sc_len = int64_t(align_up(size_t(cap), 4)) + 8;
    if (c->compact)
        for (int k = 0; k < c->n_sets; ++k)
            for (int l = 0; l < n_layers; ++l) {
                LSA_ALLOC(c->ks[k].kc[l], size_t(cap) * p.d * elem_size(p.k_dtype));
                if (p.k_dtype == LSA_E4M3) LSA_ALLOC(c->ks[k].sc[l], size_t(c->sc_len) * 4);
            }
    LSA_ALLOC(c->topk_idx, size_t(p.B) * p.topk * 4);
    LSA_ALLOC(c->topk_pos, size_t(p.B) * p.topk * 4);
    LSA_ALLOC(c->topk_cnt, size_t(p.B) * 4);
    LSA_ALLOC(c->err, 16);
    LSA_ALLOC(c->sel_ws, c->sel_ws_bytes);
    LSA_ALLOC(c->attn_ws, c->attn_ws_bytes);
    LSA_ALLOC(c->owner, size_t(cap) * 4);
    LSA_ALLOC(c->fetched, 16);
    LSA_ALLOC(c->fetch_ws, fetch_workspace(cap));
    for (auto &sg : c->stage) {
        LSA_ALLOC(sg.q, qbytes * n_layers);
        LSA_ALLOC(sg.w, size_t(n_layers) * p.B * p.H * 4);
        LSA_ALLOC(sg.Q, Qbytes);
        LSA_ALLOC(sg.out, Qbytes);
        LSA_ALLOC(sg.lse, size_t(p.B) * p.Hq * 4);
    }
#undef LSA_ALLOC
    if (s == LSA_OK) {
        cudaError_t ce = cudaMemcpy(c->seq_off_d, so, size_t(p.B + 1) * 8, cudaMemcpyHostToDevice);
        if (ce == cudaSuccess) ce = cudaMemset(c->err, 0, 16);
        if (ce == cudaSuccess) ce = cudaMemset(c->hot, 0, size_t(arena_rows) * p.row_bytes);
        if (merged) {
            // always-resident context: the last `window` entries of each sequence, then the HCA rows
            char *arena = static_cast<char *>(c->hot);
            const char *cold = static_cast<const char *>(p.cold_host);
            for (int b = 0; b < p.B && ce == cudaSuccess; ++b) {
                const int64_t w_b = std::min<int64_t>(p.window, so[b + 1] - so[b]);
                if (w_b > 0)
                    ce = cudaMemcpy(arena + (c->win_base + int64_t(b) * p.window) * p.row_bytes,
                                    cold + (so[b + 1] - w_b) * p.row_bytes, size_t(w_b) * p.row_bytes,
                                    cudaMemcpyDefault);
            }
            if (ce == cudaSuccess && n_hca > 0)
                ce = cudaMemcpy(arena + c->hca_base * p.row_bytes, p.hca_rows, size_t(n_hca) * p.row_bytes,
                                cudaMemcpyDefault);
            std::vector<int64_t> ho(p.B + 1, 0);
            if (p.hca_rows) ho.assign(p.hca_off_host, p.hca_off_host + p.B + 1);
            if (ce == cudaSuccess) ce = cudaMemcpy(c->hca_off_d, ho.data(), ho.size() * 8, cudaMemcpyHostToDevice);
        }
        // empty cache: no entry resident, no slot owned
        if (ce == cudaSuccess) ce = cudaMemset(c->slot_of, 0xFF, size_t(p.n_total > 0 ? p.n_total : 1) * 4);
        if (ce == cudaSuccess) ce = cudaMemset(c->owner, 0xFF, size_t(cap) * 4);
        if (ce == cudaSuccess) ce = cudaMemset(c->fetched, 0, 16);
        for (int k = 0; k < c->n_sets; ++k) {
            // an empty kept set: no position, no slot
            if (ce == cudaSuccess) ce = cudaMemset(c->ks[k].kept_off, 0, size_t(p.B + 1) * 8);
            if (ce == cudaSuccess) ce = cudaMemset(c->ks[k].kept_slot, 0xFF, size_t(cap) * 4);
            for (int l = 0; l < n_layers && c->compact; ++l) {
                if (ce == cudaSuccess)
                    ce = cudaMemset(c->ks[k].kc[l], 0, size_t(cap) * p.d * elem_size(p.k_dtype));
                if (ce == cudaSuccess && c->ks[k].sc[l]) ce = cudaMemset(c->ks[k].sc[l], 0, size_t(c->sc_len) * 4);
            }
        }
        if (ce == cudaSuccess) ce = cudaStreamCreateWithFlags(&c->side, cudaStreamNonBlocking);
        if (ce == cudaSuccess) ce = cudaStreamCreateWithFlags(&c->cap, cudaStreamNonBlocking);
        if (ce == cudaSuccess) ce = cudaEventCreateWithFlags(&c->ev_sel, cudaEventDisableTiming);
        if (ce == cudaSuccess) ce = cudaEventCreateWithFlags(&c->ev_gather, cudaEventDisableTiming);
        if (ce == cudaSuccess) ce = cudaEventCreateWithFlags(&c->ev_assign, cudaEventDisableTiming);
        if (ce == cudaSuccess) ce = cudaEventCreateWithFlags(&c->ev_pred, cudaEventDisableTiming);
        if (ce == cudaSuccess) ce = cudaEventCreateWithFlags(&c->ev_pend, cudaEventDisableTiming);
        if (ce == cudaSuccess) ce = cudaStreamCreateWithFlags(&c->h2d, cudaStreamNonBlocking);
        if (ce == cudaSuccess) ce = cudaStreamCreateWithFlags(&c->d2h, cudaStreamNonBlocking);
        for (auto &sg : c->stage)
            for (cudaEvent_t *e : {&sg.in_ready, &sg.used, &sg.lse_done})
                if (ce == cudaSuccess) ce = cudaEventCreateWithFlags(e, cudaEventDisableTiming);
        if (ce != cudaSuccess) {
            set_error("lsa_ctx_create: %s", cudaGetErrorString(ce));
            s = LSA_ERR_CUDA;
        }
    }
    if (s != LSA_OK) {
        free_all(c);
        delete c;
        return s;
    }
    *out = c;
    return LSA_OK;
}

lsa_status lsa_ctx_destroy(lsa_ctx *c) {
    clear_error();
    if (!c) return LSA_OK;
    cudaDeviceSynchronize();
    free_all(c);
    delete c;
    return LSA_OK;
}

lsa_status lsa_decode_step(lsa_ctx *c, int64_t t, const void *q, const float *w, const void *Q, void *out,
                           float *lse, void *stream) {
    clear_error();
    LSA_CHECK_ARG(c && q && w && Q && out, "lsa_decode_step: ctx, q, w, Q, out required");
    LSA_CHECK_ARG(t >= 0, "lsa_decode_step: t < 0");
    LSA_CHECK_ARG(aligned16(Q) && aligned16(out), "lsa_decode_step: Q and out must be 16-byte aligned");
    return run_step(c, t, q, w, Q, out, lse, as_stream(stream));
}

lsa_status lsa_decode_step_host(lsa_ctx *c, int64_t t, const void *q_host, const float *w_host,
                                const void *Q_host, void *out_host, float *lse_host, void *stream) {
    clear_error();
    LSA_CHECK_ARG(c && q_host && w_host && Q_host && out_host, "lsa_decode_step_host: ctx, q, w, Q, out required");
    LSA_CHECK_ARG(t >= 0, "lsa_decode_step_host: t < 0");
    const lsa_params &p = c->p;
    cudaStream_t st = as_stream(stream);
    const size_t qbytes = size_t(p.B) * p.H * p.d * elem_size(p.q_dtype);
    const size_t Qbytes = size_t(p.B) * p.Hq * p.D * elem_size(p.attn_dtype);
    auto &sg = c->stage[c->host_calls & 1];
    // inputs on the copy stream, once the slot's previous step has read them;
    // they overlap the kernels of the step enqueued before this one
    LSA_CUDA(cudaStreamWaitEvent(c->h2d, sg.used, 0));
    LSA_CUDA(cudaMemcpyAsync(sg.q, q_host, qbytes * c->n_layers, cudaMemcpyHostToDevice, c->h2d));
    LSA_CUDA(cudaMemcpyAsync(sg.w, w_host, size_t(c->n_layers) * p.B * p.H * 4, cudaMemcpyHostToDevice, c->h2d));
    LSA_CUDA(cudaMemcpyAsync(sg.Q, Q_host, Qbytes, cudaMemcpyHostToDevice, c->h2d));
    LSA_CUDA(cudaEventRecord(sg.in_ready, c->h2d));
    LSA_CUDA(cudaStreamWaitEvent(st, sg.in_ready, 0));
    // outputs in page-locked host memory mapped for the device: the attention writes them there
    // directly (posted writes over the host link), with no staging buffer and no copy
    void *out_map = mapped_host(out_host);
    float *lse_map = lse_host ? static_cast<float *>(mapped_host(lse_host)) : nullptr;
    const bool direct = out_map && aligned16(out_map) && (!lse_host || lse_map);
    lsa_status s = direct ? run_step(c, t, sg.q, sg.w, sg.Q, out_map, lse_map, st)
                          : run_step(c, t, sg.q, sg.w, sg.Q, sg.out, sg.lse, st);
    if (s != LSA_OK) return s;
    LSA_CUDA(cudaEventRecord(sg.used, st));
    ++c->host_calls;
    if (direct) return LSA_OK;
    // otherwise out on the caller's stream, lse beside it on the second copy
    // stream; the caller's stream joins both before it completes
    LSA_CUDA(cudaMemcpyAsync(out_host, sg.out, Qbytes, cudaMemcpyDeviceToHost, st));
    if (lse_host) {
        LSA_CUDA(cudaStreamWaitEvent(c->d2h, sg.used, 0));
        LSA_CUDA(cudaMemcpyAsync(lse_host, sg.lse, size_t(p.B) * p.Hq * 4, cudaMemcpyDeviceToHost, c->d2h));
        LSA_CUDA(cudaEventRecord(sg.lse_done, c->d2h));
        LSA_CUDA(cudaStreamWaitEvent(st, sg.lse_done, 0));
    }
    return LSA_OK;
}

lsa_status lsa_ctx_get_view(lsa_ctx *c, lsa_ctx_view *v) {
    clear_error();
    LSA_CHECK_ARG(c && v, "lsa_ctx_get_view: ctx and view required");
    v->z = c->z;
    v->z_kept = c->z_kept;
    v->kept_idx = c->ks[c->cur].kept_idx;
    v->kept_off = c->ks[c->cur].kept_off;
    v->slot_of = c->slot_of;
    v->hot = c->hot;
    v->topk_idx = c->topk_idx;
    v->topk_pos = c->topk_pos;
    v->topk_cnt = c->topk_cnt;
    v->err = c->err;
    v->kept_slot = c->p.full_fetch ? nullptr : c->ks[c->cur].kept_slot;
    v->owner = c->p.full_fetch ? nullptr : c->owner;
    v->fetched = c->fetched;
    v->attn_rows = c->attn_rows;
    v->attn_row_cap = c->row_cap;
    v->win_base = c->win_base;
    v->hca_base = c->hca_base;
    return LSA_OK;
}

lsa_status lsa_ctx_set_graphs(lsa_ctx *c, int32_t enable) {
    clear_error();
    LSA_CHECK_ARG(c, "lsa_ctx_set_graphs: ctx required");
    c->use_graphs = enable != 0;
    return LSA_OK;
}

lsa_status lsa_ctx_set_timing(lsa_ctx *c, int32_t enable) {
    clear_error();
    LSA_CHECK_ARG(c, "lsa_ctx_set_timing: ctx required");
    c->timing = enable != 0;
    return LSA_OK;
}

lsa_status lsa_ctx_stage_times(lsa_ctx *c, double *ms, int64_t *calls) {
    clear_error();
    LSA_CHECK_ARG(c && ms && calls, "lsa_ctx_stage_times: ctx, ms, calls required");
    for (auto &pe : c->pending) {
        LSA_CUDA(cudaEventSynchronize(pe.b));
        float dt = 0.f;
        LSA_CUDA(cudaEventElapsedTime(&dt, pe.a, pe.b));
        c->ms[pe.stage] += dt;
        c->calls[pe.stage] += 1;
        c->free_events.push_back(pe.a);
        c->free_events.push_back(pe.b);
    }
    c->pending.clear();
    for (int i = 0; i < LSA_STAGE_COUNT; ++i) {
        ms[i] = c->ms[i];
        calls[i] = c->calls[i];
    }
    return LSA_OK;
}

lsa_status lsa_ctx_reset_counters(lsa_ctx *c) {
    clear_error();
    LSA_CHECK_ARG(c, "lsa_ctx_reset_counters: ctx required");
    for (auto &pe : c->pending) {
        cudaEventSynchronize(pe.b);
        c->free_events.push_back(pe.a);
        c->free_events.push_back(pe.b);
    }
    c->pending.clear();
    for (int i = 0; i < LSA_STAGE_COUNT; ++i) { c->ms[i] = 0; c->calls[i] = 0; }
    c->launches = 0;
    return LSA_OK;
}

int64_t lsa_ctx_launches(lsa_ctx *c) { return c ? c->launches : -1; }

lsa_status lsa_ctx_flush_cache(lsa_ctx *c, void *stream) {
    clear_error();
    LSA_CHECK_ARG(c, "lsa_ctx_flush_cache: ctx required");
    const lsa_params &p = c->p;
    cudaStream_t st = as_stream(stream);
    // no entry resident and no slot owned: the next refresh (or prediction) fetches every kept row; the
    // current kept set's rows stay where they are (its steps keep reading them, and a prediction's fetch
    // never evicts its slots)
    LSA_CUDA(cudaMemsetAsync(c->slot_of, 0xFF, size_t(p.n_total > 0 ? p.n_total : 1) * 4, st));
    LSA_CUDA(cudaMemsetAsync(c->owner, 0xFF, size_t(p.kept_capacity) * 4, st));
    return LSA_OK;
}

}  // extern "C"
