// lq_api.cu -- the C ABI declared in include/lq_state.h: argument checks,
// workspace carving, the host-side window counter and kernel sequencing.
// Every entry point validates on the host first and launches nothing on error.
#include <stdlib.h>
#include <string.h>

#include <new>

#include "../../include/lq_state.h"
#include "lq_kernels.h"
#include "lq_prefill.h"

using lq::Layout;

struct lq_state {
    lq_config cfg;
    Layout L;
    unsigned char *ws;
    size_t bytes;
    int *status;
    int *hp_rows;
    int *slot_rows;
    float *static_ms;   // smoothing 2: [H][dk+dv] fixed key-row and value-column scales
    unsigned char *rec;
    size_t heads;
    int n;  // tokens buffered in the current window (without window phases)
    // Window phases (lq_state_set_phases): phase [B] and the batch entries
    // ordered by phase in the workspace; on the host the phases and, per phase
    // p, the range h_off[p] .. h_off[p+1] of d_order holding its entries.  The
    // window-end launches run on `side`, forked from and joined back into the
    // caller's stream by two events.
    int phased;
    long long since;   // steps since the last common window start
    int *d_phase, *d_order;
    int *h_phase, *h_off;
    cudaStream_t side;
    cudaEvent_t ev_fork, ev_join;
};

namespace {

constexpr size_t kAlign = 256;
constexpr size_t kMaxSmem = 227 * 1024;

size_t align_sz(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool is_int8(const lq_config *c) { return c->mode == LQ_MODE_INT8_STEP || c->mode == LQ_MODE_INT8_WINDOW; }

// Code width of the quantized state (0 reads as 8).
int bits_of(const lq_config *c) { return c->state_bits == 0 ? 8 : c->state_bits; }

Layout layout_of(const lq_config *c) {
    const int W = c->mode == LQ_MODE_INT8_STEP ? 1 : c->W;
    return lq::make_layout(c->dk, c->dv, c->n_hp_rows, c->r, W, c->gate == LQ_GATE_CHANNEL,
                           c->mode == LQ_MODE_INT8_WINDOW && c->buffer_bf16 == 1, bits_of(c));
}

int check_codec_fields(const lq_config *c) {
    if (c->dk != 64 && c->dk != 128) return LQ_ERR_UNSUPPORTED;
    if (c->dv != 64 && c->dv != 128) return LQ_ERR_UNSUPPORTED;
    const int bits = bits_of(c);
    if (bits != 8 && bits != 6 && bits != 4) return LQ_ERR_INVALID_ARG;
    if (bits != 8 && c->n_hp_rows > 0) return LQ_ERR_UNSUPPORTED;   // packed codes: no BF16 rows
    if (c->r < 0 || c->r > (c->dk < c->dv ? c->dk : c->dv)) return LQ_ERR_INVALID_ARG;
    if (c->power_iters < 0 || c->power_iters > 1000) return LQ_ERR_INVALID_ARG;
    if (c->n_hp_rows < 0 || c->n_hp_rows >= c->dk) return LQ_ERR_INVALID_ARG;
    if (c->smoothing < 0 || c->smoothing > 2) return LQ_ERR_INVALID_ARG;
    if (c->smoothing == 2 && c->n_hp_rows > 0) return LQ_ERR_UNSUPPORTED;   // static scales: no BF16 rows
    return LQ_OK;
}

int check_config(const lq_config *c) {
    if (!c) return LQ_ERR_INVALID_ARG;
    if (c->B < 1 || c->H < 1 || c->Hk < 1) return LQ_ERR_SHAPE;
    if (c->Hk > c->H || c->H % c->Hk != 0) return LQ_ERR_SHAPE;
    if ((long long)c->B * c->H > (1ll << 31) - 1) return LQ_ERR_SHAPE;
    if (c->gate != LQ_GATE_SCALAR && c->gate != LQ_GATE_CHANNEL) return LQ_ERR_INVALID_ARG;
    if (c->mode != LQ_MODE_FP32 && c->mode != LQ_MODE_INT8_STEP && c->mode != LQ_MODE_INT8_WINDOW)
        return LQ_ERR_INVALID_ARG;
    if (c->fused_flush != 0 && c->fused_flush != 1) return LQ_ERR_INVALID_ARG;
    if (c->buffer_bf16 != 0 && c->buffer_bf16 != 1) return LQ_ERR_INVALID_ARG;
    if (c->buffer_bf16 == 1 && c->mode != LQ_MODE_INT8_WINDOW) return LQ_ERR_INVALID_ARG;
    if (c->buffer_bf16 == 1 && c->n_hp_rows > 0) return LQ_ERR_UNSUPPORTED;   // not built with BF16 rows
    if (c->mode == LQ_MODE_FP32 && c->state_bits != 0 && c->state_bits != 8) return LQ_ERR_INVALID_ARG;
    if (c->mode == LQ_MODE_FP32 && c->smoothing == 2) return LQ_ERR_INVALID_ARG;
    int rc = check_codec_fields(c);
    if (rc) return rc;
    if (is_int8(c)) {
        if (c->W < 1) return LQ_ERR_INVALID_ARG;
        if (c->W > LQ_MAX_WINDOW) return LQ_ERR_UNSUPPORTED;
        if (c->mode == LQ_MODE_INT8_STEP && c->W != 1) return LQ_ERR_INVALID_ARG;
        if (lq::decode_smem_bytes(c->dk, c->dv, layout_of(c)) > kMaxSmem) return LQ_ERR_UNSUPPORTED;
    } else if (c->n_hp_rows != 0) {
        return LQ_ERR_INVALID_ARG;
    }
    return LQ_OK;
}

size_t hp_bytes(const lq_config *c) { return align_sz((size_t)c->H * c->n_hp_rows * 4, kAlign); }

size_t slot_bytes(const lq_config *c) {
    return c->n_hp_rows > 0 ? align_sz((size_t)c->H * c->dk * 4, kAlign) : 0;
}

size_t static_bytes(const lq_config *c) {
    return c->smoothing == 2 ? align_sz((size_t)c->H * (c->dk + c->dv) * 4, kAlign) : 0;
}

// Window mode: the phase array and the phase-ordered batch entries.
size_t phase_bytes(const lq_config *c) {
    return c->mode == LQ_MODE_INT8_WINDOW ? align_sz((size_t)2 * c->B * 4, kAlign) : 0;
}

size_t record_bytes(const lq_config *c) {
    if (is_int8(c)) return (size_t)layout_of(c).rec_bytes;
    return (size_t)c->dk * c->dv * 4;
}

int check_hp_rows(const lq_config *c, const int32_t *rows) {
    if (c->n_hp_rows == 0) return LQ_OK;
    if (!rows) return LQ_ERR_INVALID_ARG;
    for (int h = 0; h < c->H; ++h) {
        const int32_t *r = rows + (size_t)h * c->n_hp_rows;
        for (int p = 0; p < c->n_hp_rows; ++p) {
            if (r[p] < 0 || r[p] >= c->dk) return LQ_ERR_INVALID_ARG;
            for (int q = 0; q < p; ++q)
                if (r[q] == r[p]) return LQ_ERR_INVALID_ARG;
        }
    }
    return LQ_OK;
}

lq::QPtrs record_ptrs(const lq_state *st) {
    const Layout &L = st->L;
    lq::QPtrs q{};
    const size_t hs = (size_t)L.rec_bytes;
    q.codes = st->rec + L.off_codes; q.codes_hs = hs; q.codes_t = L.P == 0 ? 1 : 0;
    q.hp = st->rec + L.off_hp; q.hp_hs = hs;
    q.m = st->rec + L.off_m; q.m_hs = hs;
    q.s = st->rec + L.off_s; q.s_hs = hs;
    q.ck = st->rec + L.off_ent; q.ck_hs = hs; q.ck_js = L.dk + L.dv;
    q.cw = st->rec + L.off_ent + (size_t)L.dk * 4; q.cw_hs = hs; q.cw_js = L.dk + L.dv;
    q.gam = st->rec + L.off_gam; q.gam_hs = hs; q.gam_n = L.kda ? 2 * L.dk : 2;   // G and sigma
    return q;
}

lq::QPtrs view_ptrs(const lq_config *c, const lq_qstate_view *v) {
    lq::QPtrs q{};
    const int dk = c->dk, dv = c->dv, P = c->n_hp_rows, r = c->r;
    q.codes = reinterpret_cast<unsigned char *>(v->codes); q.codes_hs = (size_t)(dk - P) * dv;
    q.hp = reinterpret_cast<unsigned char *>(v->bf16_rows); q.hp_hs = (size_t)P * dv * 2;
    q.m = reinterpret_cast<unsigned char *>(v->m); q.m_hs = (size_t)dk * 4;
    q.s = reinterpret_cast<unsigned char *>(v->s); q.s_hs = (size_t)dv * 4;
    q.ck = reinterpret_cast<unsigned char *>(v->comp_k); q.ck_hs = (size_t)r * dk * 4; q.ck_js = dk;
    q.cw = reinterpret_cast<unsigned char *>(v->comp_v); q.cw_hs = (size_t)r * dv * 4; q.cw_js = dv;
    return q;
}

int check_view(const lq_config *c, const lq_qstate_view *v) {
    if (!v || !v->codes || !v->m || !v->s) return LQ_ERR_INVALID_ARG;
    if (c->n_hp_rows > 0 && !v->bf16_rows) return LQ_ERR_INVALID_ARG;
    if (c->r > 0 && (!v->comp_k || !v->comp_v)) return LQ_ERR_INVALID_ARG;
    const uintptr_t a = reinterpret_cast<uintptr_t>(v->codes) | reinterpret_cast<uintptr_t>(v->m) |
                        reinterpret_cast<uintptr_t>(v->s) | reinterpret_cast<uintptr_t>(v->bf16_rows) |
                        reinterpret_cast<uintptr_t>(v->comp_k) | reinterpret_cast<uintptr_t>(v->comp_v);
    if (a & 15) return LQ_ERR_INVALID_ARG;  // 16-byte vector access
    return LQ_OK;
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? LQ_OK : LQ_ERR_CUDA; }

lq::DecodeArgs decode_args(const lq_state *st) {
    lq::DecodeArgs a{};
    a.L = st->L;
    a.rec = st->rec;
    a.B = st->cfg.B; a.H = st->cfg.H; a.Hk = st->cfg.Hk;
    a.K = st->cfg.power_iters;
    a.smoothing = st->cfg.smoothing;
    a.n = st->n;
    a.hp_rows = st->hp_rows;
    a.slot_rows = st->slot_rows;
    a.status = st->status;
    if (st->phased) {
        const int W = st->L.W;
        a.phase = st->d_phase;
        a.n = st->since < W ? (int)st->since : W;
        a.nmod = (int)(st->since % W);
    }
    return a;
}

// Tokens batch entry b holds (every entry without phases).
int entry_buffered(const lq_state *st, int phase) {
    if (!st->phased) return st->n;
    const int W = st->L.W;
    const long long p = (st->since + phase) % W;
    return (int)(p < st->since ? p : st->since);
}

// The most tokens any batch entry holds: 0 iff every entry is at a window start.
int buffered_max(const lq_state *st) {
    if (!st->phased) return st->n;
    int m = 0;
    for (int p = 0; p < st->L.W; ++p)
        if (st->h_off[p + 1] > st->h_off[p]) {
            const int v = entry_buffered(st, p);
            m = v > m ? v : m;
        }
    return m;
}

void release(lq_state *st) {
    if (st->side) {
        cudaEventDestroy(st->ev_fork);
        cudaEventDestroy(st->ev_join);
        cudaStreamDestroy(st->side);
    }
    free(st->h_phase);
    free(st->h_off);
    delete st;
}

}  // namespace

extern "C" {

int lq_config_check(const lq_config *cfg) { return check_config(cfg); }

size_t lq_workspace_bytes(const lq_config *cfg) {
    if (check_config(cfg) != LQ_OK) return 0;
    return kAlign + hp_bytes(cfg) + slot_bytes(cfg) + static_bytes(cfg) + phase_bytes(cfg) +
           (size_t)cfg->B * cfg->H * record_bytes(cfg);
}

static int state_init(lq_state **out, const lq_config *cfg, void *d_workspace, size_t bytes, const float *d_S0,
                      const int32_t *h_hp_row_ids, const float *d_static_m, const float *d_static_s, void *stream) {
    if (!out) return LQ_ERR_INVALID_ARG;
    *out = nullptr;
    int rc = check_config(cfg);
    if (rc) return rc;
    if ((cfg->smoothing == 2) != (d_static_m != nullptr)) return LQ_ERR_INVALID_ARG;
    if (cfg->smoothing == 2 && !d_static_s) return LQ_ERR_INVALID_ARG;
    if (!d_workspace || !d_S0) return LQ_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(d_workspace) % kAlign) return LQ_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(d_S0) % 16) return LQ_ERR_INVALID_ARG;
    if (bytes < lq_workspace_bytes(cfg)) return LQ_ERR_WORKSPACE;
    rc = check_hp_rows(cfg, h_hp_row_ids);
    if (rc) return rc;
    lq_state *st = new (std::nothrow) lq_state;
    if (!st) return LQ_ERR_INVALID_ARG;
    st->cfg = *cfg;
    if (cfg->mode == LQ_MODE_INT8_STEP) st->cfg.W = 1;
    st->L = layout_of(cfg);
    st->ws = static_cast<unsigned char *>(d_workspace);
    st->bytes = bytes;
    st->status = reinterpret_cast<int *>(st->ws);
    st->hp_rows = reinterpret_cast<int *>(st->ws + kAlign);
    st->slot_rows = reinterpret_cast<int *>(st->ws + kAlign + hp_bytes(cfg));
    st->static_ms = cfg->smoothing == 2
                        ? reinterpret_cast<float *>(st->ws + kAlign + hp_bytes(cfg) + slot_bytes(cfg))
                        : nullptr;
    st->d_phase = reinterpret_cast<int *>(st->ws + kAlign + hp_bytes(cfg) + slot_bytes(cfg) + static_bytes(cfg));
    st->d_order = st->d_phase + cfg->B;
    st->rec = st->ws + kAlign + hp_bytes(cfg) + slot_bytes(cfg) + static_bytes(cfg) + phase_bytes(cfg);
    st->heads = (size_t)cfg->B * cfg->H;
    st->n = 0;
    st->phased = 0;
    st->since = 0;
    st->h_phase = st->h_off = nullptr;
    st->side = nullptr;
    st->ev_fork = st->ev_join = nullptr;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // Per head: the key row of every INT8 slot (increasing), then of every BF16 row.
    int32_t *slots = nullptr;
    if (cfg->n_hp_rows > 0) {
        slots = static_cast<int32_t *>(malloc((size_t)cfg->H * cfg->dk * 4));
        if (!slots) {
            delete st;
            return LQ_ERR_INVALID_ARG;
        }
        for (int h = 0; h < cfg->H; ++h) {
            const int32_t *hr = h_hp_row_ids + (size_t)h * cfg->n_hp_rows;
            int32_t *out_h = slots + (size_t)h * cfg->dk;
            int j = 0;
            for (int i = 0; i < cfg->dk; ++i) {
                bool hp = false;
                for (int p = 0; p < cfg->n_hp_rows; ++p) hp = hp || hr[p] == i;
                if (!hp) out_h[j++] = i;
            }
            for (int p = 0; p < cfg->n_hp_rows; ++p) out_h[j++] = hr[p];
        }
    }
    cudaError_t e = cudaMemsetAsync(st->status, 0, sizeof(int), s);
    if (e == cudaSuccess && cfg->n_hp_rows > 0)
        e = cudaMemcpyAsync(st->hp_rows, h_hp_row_ids, (size_t)cfg->H * cfg->n_hp_rows * 4,
                            cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && cfg->n_hp_rows > 0)
        e = cudaMemcpyAsync(st->slot_rows, slots, (size_t)cfg->H * cfg->dk * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && st->static_ms) {   // [H][dk] and [H][dv] -> [H][dk+dv]
        const size_t pitch = (size_t)(cfg->dk + cfg->dv) * 4;
        e = cudaMemcpy2DAsync(st->static_ms, pitch, d_static_m, (size_t)cfg->dk * 4, (size_t)cfg->dk * 4, cfg->H,
                              cudaMemcpyDeviceToDevice, s);
        if (e == cudaSuccess)
            e = cudaMemcpy2DAsync(st->static_ms + cfg->dk, pitch, d_static_s, (size_t)cfg->dv * 4,
                                  (size_t)cfg->dv * 4, cfg->H, cudaMemcpyDeviceToDevice, s);
    }
    if (e == cudaSuccess) {
        if (is_int8(cfg)) {
            lq::CodecArgs a{};
            a.H = cfg->H; a.r = cfg->r; a.K = cfg->power_iters; a.smoothing = cfg->smoothing;
            a.P = cfg->n_hp_rows; a.hp_rows = st->hp_rows; a.S_in = d_S0; a.bits = bits_of(cfg);
            a.static_ms = st->static_ms;
            a.q = record_ptrs(st);
            a.status = st->status;
            e = lq::launch_quantize(a, cfg->dk, cfg->dv, (int)st->heads, s);
        } else {
            e = cudaMemcpyAsync(st->rec, d_S0, st->heads * record_bytes(cfg), cudaMemcpyDeviceToDevice, s);
        }
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    free(slots);
    if (e != cudaSuccess) {
        delete st;
        return LQ_ERR_CUDA;
    }
    *out = st;
    return LQ_OK;
}

int lq_state_init(lq_state **out, const lq_config *cfg, void *d_workspace, size_t bytes, const float *d_S0,
                  const int32_t *h_hp_row_ids, void *stream) {
    return state_init(out, cfg, d_workspace, bytes, d_S0, h_hp_row_ids, nullptr, nullptr, stream);
}

int lq_state_init_static(lq_state **out, const lq_config *cfg, void *d_workspace, size_t bytes, const float *d_S0,
                         const float *d_static_m, const float *d_static_s, void *stream) {
    if (!d_static_m || !d_static_s) return LQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d_static_m) | reinterpret_cast<uintptr_t>(d_static_s)) & 3)
        return LQ_ERR_INVALID_ARG;
    return state_init(out, cfg, d_workspace, bytes, d_S0, nullptr, d_static_m, d_static_s, stream);
}

int lq_decode_step(lq_state *st, const float *d_q, const float *d_k, const float *d_v, const float *d_beta,
                   const float *d_alpha, float *d_o, void *stream) {
    if (!st || !d_q || !d_k || !d_v || !d_beta || !d_alpha || !d_o) return LQ_ERR_INVALID_ARG;
    const lq_config &c = st->cfg;
    // q, k, v and a per-channel gate are fetched with 16-byte bulk copies.
    const uintptr_t al = reinterpret_cast<uintptr_t>(d_q) | reinterpret_cast<uintptr_t>(d_k) |
                         reinterpret_cast<uintptr_t>(d_v) |
                         (c.gate == LQ_GATE_CHANNEL ? reinterpret_cast<uintptr_t>(d_alpha) : 0);
    if (al & 15) return LQ_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool kda = c.gate == LQ_GATE_CHANNEL;
    if (c.mode == LQ_MODE_FP32) {
        lq::Fp32Args a{};
        a.S = reinterpret_cast<float *>(st->rec);
        a.B = c.B; a.H = c.H; a.Hk = c.Hk;
        a.q = d_q; a.k = d_k; a.v = d_v; a.beta = d_beta; a.alpha = d_alpha; a.o = d_o;
        a.status = st->status;
        return cuda_rc(lq::launch_fp32_step(a, c.dk, c.dv, (int)st->heads, kda, s));
    }
    lq::DecodeArgs a = decode_args(st);
    a.q = d_q; a.k = d_k; a.v = d_v; a.beta = d_beta; a.alpha = d_alpha; a.o = d_o;
    const bool damp = c.n_hp_rows > 0;
    if (st->phased) {
        // The entries whose window ends at this step (phase W - 1 - since mod
        // W) take the window-end kernel on the side stream, the others the
        // buffering kernel (which skips the former) on `stream`.
        const int W = st->L.W;
        const int rho = W - 1 - a.nmod;
        const int first = st->h_off[rho], cnt = st->h_off[rho + 1] - first;
        cudaError_t e = cudaSuccess;
        if (cnt > 0) {
            e = cudaEventRecord(st->ev_fork, s);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(st->side, st->ev_fork, 0);
            lq::DecodeArgs af = a;
            af.flush_list = st->d_order + first;
            if (e == cudaSuccess) e = lq::launch_decode(af, c.dk, c.dv, cnt * c.H, kda, true, damp, st->side);
        }
        if (e == cudaSuccess && cnt < c.B) e = lq::launch_decode(a, c.dk, c.dv, (int)st->heads, kda, false, damp, s);
        if (e == cudaSuccess && cnt > 0) {
            e = cudaEventRecord(st->ev_join, st->side);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(s, st->ev_join, 0);
        }
        if (e == cudaSuccess) st->since += 1;
        return cuda_rc(e);
    }
    if (st->n >= st->L.W) return LQ_ERR_WINDOW_FULL;
    const bool flush = (c.mode == LQ_MODE_INT8_STEP) || (c.fused_flush && st->n + 1 == st->L.W);
    const int rc = cuda_rc(lq::launch_decode(a, c.dk, c.dv, (int)st->heads, kda, flush, damp, s));
    if (rc == LQ_OK) st->n = flush ? 0 : st->n + 1;
    return rc;
}

int lq_state_set_phases(lq_state *st, const int32_t *h_phase, void *stream) {
    if (!st) return LQ_ERR_INVALID_ARG;
    const lq_config &c = st->cfg;
    if (c.mode != LQ_MODE_INT8_WINDOW || c.fused_flush != 1) return LQ_ERR_UNSUPPORTED;
    if (buffered_max(st) > 0) return LQ_ERR_UNSUPPORTED;
    const int W = st->L.W;
    if (!h_phase) {
        st->phased = 0;
        st->n = 0;
        return LQ_OK;
    }
    for (int b = 0; b < c.B; ++b)
        if (h_phase[b] < 0 || h_phase[b] >= W) return LQ_ERR_INVALID_ARG;
    int *ph = static_cast<int *>(malloc((size_t)c.B * sizeof(int)));
    int *off = static_cast<int *>(calloc((size_t)W + 1, sizeof(int)));
    int *order = static_cast<int *>(malloc((size_t)c.B * sizeof(int)));
    if (!ph || !off || !order) {
        free(ph); free(off); free(order);
        return LQ_ERR_INVALID_ARG;
    }
    // counting sort of the entries by phase
    for (int b = 0; b < c.B; ++b) {
        ph[b] = h_phase[b];
        off[ph[b] + 1] += 1;
    }
    for (int p = 0; p < W; ++p) off[p + 1] += off[p];
    {
        int *fill = static_cast<int *>(malloc((size_t)W * sizeof(int)));
        if (!fill) {
            free(ph); free(off); free(order);
            return LQ_ERR_INVALID_ARG;
        }
        memcpy(fill, off, (size_t)W * sizeof(int));
        for (int b = 0; b < c.B; ++b) order[fill[ph[b]]++] = b;
        free(fill);
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (!st->side) {
        int least = 0, greatest = 0;
        e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
        if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&st->side, cudaStreamNonBlocking, greatest);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&st->ev_fork, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&st->ev_join, cudaEventDisableTiming);
    }
    if (e == cudaSuccess) e = cudaMemcpyAsync(st->d_phase, ph, (size_t)c.B * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(st->d_order, order, (size_t)c.B * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    free(order);
    if (e != cudaSuccess) {
        free(ph); free(off);
        return LQ_ERR_CUDA;
    }
    free(st->h_phase);
    free(st->h_off);
    st->h_phase = ph;
    st->h_off = off;
    st->phased = 1;
    st->since = 0;
    st->n = 0;
    return LQ_OK;
}

int lq_window_flush(lq_state *st, void *stream) {
    if (!st) return LQ_ERR_INVALID_ARG;
    if (st->cfg.mode != LQ_MODE_INT8_WINDOW) return LQ_OK;
    if (buffered_max(st) == 0) {
        st->since = 0;   // (window phases: the schedule restarts all the same)
        return LQ_OK;
    }
    // (window phases: entries with nothing buffered leave the launch at once)
    lq::DecodeArgs a = decode_args(st);
    const int rc = cuda_rc(lq::launch_flush(a, st->cfg.dk, st->cfg.dv, (int)st->heads,
                                            st->cfg.gate == LQ_GATE_CHANNEL, st->cfg.n_hp_rows > 0, false,
                                            static_cast<cudaStream_t>(stream)));
    if (rc == LQ_OK) {
        st->n = 0;
        st->since = 0;
    }
    return rc;
}

int lq_state_buffered(const lq_state *st) { return st ? buffered_max(st) : 0; }

int lq_state_export_fp32(const lq_state *st, float *d_S, void *stream) {
    if (!st || !d_S) return LQ_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(d_S) % 16) return LQ_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (st->cfg.mode == LQ_MODE_FP32)
        return cuda_rc(cudaMemcpyAsync(d_S, st->rec, st->heads * record_bytes(&st->cfg), cudaMemcpyDeviceToDevice, s));
    lq::DecodeArgs a = decode_args(st);
    a.S_out = d_S;
    return cuda_rc(lq::launch_flush(a, st->cfg.dk, st->cfg.dv, (int)st->heads, st->cfg.gate == LQ_GATE_CHANNEL,
                                    st->cfg.n_hp_rows > 0, true, s));
}

int lq_state_export_view(const lq_state *st, const lq_qstate_view *out, void *stream) {
    if (!st) return LQ_ERR_INVALID_ARG;
    if (!is_int8(&st->cfg)) return LQ_ERR_INVALID_ARG;
    // mid-window the record's compensators may carry the decay guard's
    // rescaling; the window-start view is only whole at a window boundary
    if (buffered_max(st) > 0) return LQ_ERR_UNSUPPORTED;
    int rc = check_view(&st->cfg, out);
    if (rc) return rc;
    lq::CodecArgs a{};
    a.H = st->cfg.H; a.r = st->cfg.r; a.P = st->cfg.n_hp_rows; a.bits = bits_of(&st->cfg);
    a.q = record_ptrs(st);
    a.q.gam = nullptr;
    a.q2 = view_ptrs(&st->cfg, out);
    return cuda_rc(lq::launch_qcopy(a, st->cfg.dk, st->cfg.dv, (int)st->heads, static_cast<cudaStream_t>(stream)));
}

int lq_state_import_view(lq_state *st, const lq_qstate_view *in, void *stream) {
    if (!st) return LQ_ERR_INVALID_ARG;
    if (!is_int8(&st->cfg)) return LQ_ERR_INVALID_ARG;
    // with window phases the schedule goes on: every entry must be at a window start
    if (st->phased && buffered_max(st) > 0) return LQ_ERR_UNSUPPORTED;
    int rc = check_view(&st->cfg, in);
    if (rc) return rc;
    lq::CodecArgs a{};
    a.H = st->cfg.H; a.r = st->cfg.r; a.P = st->cfg.n_hp_rows; a.bits = bits_of(&st->cfg);
    a.q = view_ptrs(&st->cfg, in);
    a.q2 = record_ptrs(st);
    rc = cuda_rc(lq::launch_qcopy(a, st->cfg.dk, st->cfg.dv, (int)st->heads, static_cast<cudaStream_t>(stream)));
    if (rc == LQ_OK) st->n = 0;
    return rc;
}

static int codec_common(const lq_config *cfg, const int32_t *h_rows, lq::CodecArgs &a, int **d_rows,
                        cudaStream_t s) {
    if (!cfg) return LQ_ERR_INVALID_ARG;
    if (cfg->B < 1 || cfg->H < 1) return LQ_ERR_SHAPE;
    int rc = check_codec_fields(cfg);
    if (rc) return rc;
    rc = check_hp_rows(cfg, h_rows);
    if (rc) return rc;
    a.H = cfg->H; a.r = cfg->r; a.K = cfg->power_iters; a.smoothing = cfg->smoothing; a.P = cfg->n_hp_rows;
    a.bits = bits_of(cfg);
    *d_rows = nullptr;
    if (cfg->n_hp_rows > 0) {
        const size_t nb = (size_t)cfg->H * cfg->n_hp_rows * 4;
        if (cudaMallocAsync(reinterpret_cast<void **>(d_rows), nb, s) != cudaSuccess) return LQ_ERR_CUDA;
        if (cudaMemcpyAsync(*d_rows, h_rows, nb, cudaMemcpyHostToDevice, s) != cudaSuccess) {
            cudaFreeAsync(*d_rows, s);
            return LQ_ERR_CUDA;
        }
        a.hp_rows = *d_rows;
    }
    return LQ_OK;
}

int lq_quantize_state(const lq_config *cfg, const float *d_S, const int32_t *h_hp_row_ids, lq_qstate_view *out,
                      void *stream) {
    if (!d_S || (reinterpret_cast<uintptr_t>(d_S) % 16)) return LQ_ERR_INVALID_ARG;
    if (!cfg) return LQ_ERR_INVALID_ARG;
    if (cfg->smoothing == 2) return LQ_ERR_UNSUPPORTED;   // fixed scales live in a decode state
    int rc = check_view(cfg, out);
    if (rc) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    lq::CodecArgs a{};
    int *d_rows = nullptr;
    rc = codec_common(cfg, h_hp_row_ids, a, &d_rows, s);
    if (rc) return rc;
    a.S_in = d_S;
    a.q = view_ptrs(cfg, out);
    rc = cuda_rc(lq::launch_quantize(a, cfg->dk, cfg->dv, cfg->B * cfg->H, s));
    if (d_rows) cudaFreeAsync(d_rows, s);
    return rc;
}

// Row lists of lq_quantize_state_static: a fixed device array instead of a
// per-call allocation.  Host code must not use the symbol itself as a device
// address; the address is looked up once per device with that device current.
static __device__ __align__(256) int32_t g_static_rows[LQ_STATIC_ROWS_MAX];

static int static_rows_ptr(int32_t **out) {
    constexpr int kMaxDev = 64;
    static int32_t *ptr[kMaxDev] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return LQ_ERR_CUDA;
    if (!ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_rows) != cudaSuccess || !p) return LQ_ERR_CUDA;
        ptr[dev] = static_cast<int32_t *>(p);
    }
    *out = ptr[dev];
    return LQ_OK;
}

int lq_quantize_state_static(const lq_config *cfg, const float *d_S, const int32_t *h_hp_row_ids,
                             lq_qstate_view *out, void *stream) {
    // the same checks in the same order as lq_quantize_state, then the size
    // of the fixed row-list array
    if (!d_S || (reinterpret_cast<uintptr_t>(d_S) % 16)) return LQ_ERR_INVALID_ARG;
    if (!cfg) return LQ_ERR_INVALID_ARG;
    if (cfg->smoothing == 2) return LQ_ERR_UNSUPPORTED;
    int rc = check_view(cfg, out);
    if (rc) return rc;
    if (cfg->B < 1 || cfg->H < 1) return LQ_ERR_SHAPE;
    rc = check_codec_fields(cfg);
    if (rc) return rc;
    rc = check_hp_rows(cfg, h_hp_row_ids);
    if (rc) return rc;
    if ((long long)cfg->H * cfg->n_hp_rows > LQ_STATIC_ROWS_MAX) return LQ_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    lq::CodecArgs a{};
    a.H = cfg->H; a.r = cfg->r; a.K = cfg->power_iters; a.smoothing = cfg->smoothing; a.P = cfg->n_hp_rows;
    a.bits = bits_of(cfg);
    if (cfg->n_hp_rows > 0) {
        int32_t *rows = nullptr;
        rc = static_rows_ptr(&rows);
        if (rc) return rc;
        // Every entry the kernel reads is written here; nothing needs clearing.
        if (cudaMemcpyAsync(rows, h_hp_row_ids, (size_t)cfg->H * cfg->n_hp_rows * 4, cudaMemcpyHostToDevice, s) !=
            cudaSuccess)
            return LQ_ERR_CUDA;
        a.hp_rows = rows;
    }
    a.S_in = d_S;
    a.q = view_ptrs(cfg, out);
    return cuda_rc(lq::launch_quantize(a, cfg->dk, cfg->dv, cfg->B * cfg->H, s));
}

int lq_dequantize_state(const lq_config *cfg, const lq_qstate_view *in, const int32_t *h_hp_row_ids, float *d_S,
                        void *stream) {
    if (!d_S || (reinterpret_cast<uintptr_t>(d_S) % 16)) return LQ_ERR_INVALID_ARG;
    if (!cfg) return LQ_ERR_INVALID_ARG;
    int rc = check_view(cfg, in);
    if (rc) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    lq::CodecArgs a{};
    int *d_rows = nullptr;
    rc = codec_common(cfg, h_hp_row_ids, a, &d_rows, s);
    if (rc) return rc;
    a.S_out = d_S;
    a.q = view_ptrs(cfg, in);
    rc = cuda_rc(lq::launch_dequantize(a, cfg->dk, cfg->dv, cfg->B * cfg->H, s));
    if (d_rows) cudaFreeAsync(d_rows, s);
    return rc;
}

int lq_damp_select(const lq_config *cfg, int32_t n_states, const float *d_states, int32_t n_gate_samples,
                   const float *d_gates, double *d_energy, int32_t *d_rows, void *stream) {
    if (!cfg || !d_states || !d_gates || !d_energy || !d_rows) return LQ_ERR_INVALID_ARG;
    if (n_states < 1 || n_gate_samples < 1) return LQ_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(d_states) % 16) return LQ_ERR_INVALID_ARG;
    if (cfg->H < 1) return LQ_ERR_SHAPE;
    if (cfg->gate != LQ_GATE_SCALAR && cfg->gate != LQ_GATE_CHANNEL) return LQ_ERR_INVALID_ARG;
    int rc = check_codec_fields(cfg);
    if (rc) return rc;
    if (cfg->n_hp_rows < 1) return LQ_ERR_INVALID_ARG;
    if (bits_of(cfg) != 8) return LQ_ERR_UNSUPPORTED;   // the selection scores INT8 error energy
    if (cfg->smoothing == 2) return LQ_ERR_UNSUPPORTED;
    lq::CodecArgs a{};
    a.H = cfg->H; a.r = cfg->r; a.K = cfg->power_iters; a.smoothing = cfg->smoothing; a.P = cfg->n_hp_rows;
    a.bits = 8;
    a.S_in = d_states;
    a.n_states = n_states;
    a.n_gate_samples = n_gate_samples;
    a.gate_per_channel = cfg->gate == LQ_GATE_CHANNEL;
    a.gates = d_gates;
    a.energy = d_energy;
    a.rows_out = d_rows;
    return cuda_rc(lq::launch_damp_select(a, cfg->dk, cfg->dv, static_cast<cudaStream_t>(stream)));
}

int lq_fit_static_scales(const lq_config *cfg, int32_t n_states, const float *d_states, int32_t n_gate_samples,
                         const float *d_gates, float *d_m, float *d_s, void *stream) {
    if (!cfg || !d_states || !d_m || !d_s || n_states < 1) return LQ_ERR_INVALID_ARG;
    if (cfg->H < 1) return LQ_ERR_SHAPE;
    if (reinterpret_cast<uintptr_t>(d_states) % 16) return LQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d_m) | reinterpret_cast<uintptr_t>(d_s)) & 3) return LQ_ERR_INVALID_ARG;
    if (d_gates && ((reinterpret_cast<uintptr_t>(d_gates) & 3) || n_gate_samples < 1)) return LQ_ERR_INVALID_ARG;
    if (cfg->gate != LQ_GATE_SCALAR && cfg->gate != LQ_GATE_CHANNEL) return LQ_ERR_INVALID_ARG;
    int rc = check_codec_fields(cfg);
    if (rc) return rc;
    if (cfg->n_hp_rows != 0) return LQ_ERR_UNSUPPORTED;
    if ((long long)n_states * cfg->H > (1ll << 31) - 1) return LQ_ERR_SHAPE;
    lq::CodecArgs a{};
    a.H = cfg->H; a.r = cfg->r; a.K = cfg->power_iters; a.bits = bits_of(cfg);
    a.S_in = d_states;
    a.gates = d_gates;
    a.n_gate_samples = d_gates ? n_gate_samples : 0;
    a.gate_per_channel = cfg->gate == LQ_GATE_CHANNEL;
    return cuda_rc(lq::launch_fit_static(a, cfg->dk, cfg->dv, n_states, d_m, d_s, static_cast<cudaStream_t>(stream)));
}

int lq_prefill(const lq_config *cfg, int32_t T, const float *d_q, const float *d_k, const float *d_v,
               const float *d_beta, const float *d_alpha, const float *d_S0, float *d_S_out, float *d_o,
               void *stream) {
    if (!cfg || !d_S_out || T < 0 || T > (1 << 30)) return LQ_ERR_INVALID_ARG;
    if (cfg->B < 1 || cfg->H < 1 || cfg->Hk < 1) return LQ_ERR_SHAPE;
    if (cfg->Hk > cfg->H || cfg->H % cfg->Hk != 0) return LQ_ERR_SHAPE;
    if ((long long)cfg->B * cfg->H > (1ll << 31) - 1) return LQ_ERR_SHAPE;
    if (cfg->gate != LQ_GATE_SCALAR && cfg->gate != LQ_GATE_CHANNEL) return LQ_ERR_INVALID_ARG;
    if (cfg->dk != 64 && cfg->dk != 128) return LQ_ERR_UNSUPPORTED;
    if (cfg->dv != 64 && cfg->dv != 128) return LQ_ERR_UNSUPPORTED;
    if (T > 0 && (!d_q || !d_k || !d_v || !d_beta || !d_alpha)) return LQ_ERR_INVALID_ARG;
    const uintptr_t al = reinterpret_cast<uintptr_t>(d_q) | reinterpret_cast<uintptr_t>(d_k) |
                         reinterpret_cast<uintptr_t>(d_v) | reinterpret_cast<uintptr_t>(d_beta) |
                         reinterpret_cast<uintptr_t>(d_alpha) | reinterpret_cast<uintptr_t>(d_S0) |
                         reinterpret_cast<uintptr_t>(d_S_out) | reinterpret_cast<uintptr_t>(d_o);
    if (al & 3) return LQ_ERR_INVALID_ARG;
    lq::PrefillArgs a{};
    a.B = cfg->B; a.H = cfg->H; a.Hk = cfg->Hk; a.T = T;
    a.q = d_q; a.k = d_k; a.v = d_v; a.beta = d_beta; a.alpha = d_alpha;
    a.S0 = d_S0; a.S_out = d_S_out; a.o = d_o; a.status = nullptr;
    return cuda_rc(lq::launch_prefill(a, cfg->dk, cfg->dv, cfg->B * cfg->H, cfg->gate == LQ_GATE_CHANNEL,
                                      static_cast<cudaStream_t>(stream)));
}

int lq_selftest_division(const float *d_a, const float *d_b, float *d_fast, float *d_pair, float *d_ieee,
                         int32_t n, void *stream) {
    if (n < 0 || (n & 1)) return LQ_ERR_INVALID_ARG;
    if (n > 0 && (!d_a || !d_b || !d_fast || !d_pair || !d_ieee)) return LQ_ERR_INVALID_ARG;
    return cuda_rc(lq::launch_div_selftest(d_a, d_b, d_fast, d_pair, d_ieee, n, static_cast<cudaStream_t>(stream)));
}

int lq_selftest_wait(lq_state *st, int64_t limit_ns, void *stream) {
    if (!st || limit_ns < 1000 || limit_ns > 1000000000) return LQ_ERR_INVALID_ARG;
    return cuda_rc(lq::launch_wait_selftest(st->rec, st->status, (unsigned long long)limit_ns,
                                            static_cast<cudaStream_t>(stream)));
}

int lq_get_status(lq_state *st, void *stream) {
    if (!st) return LQ_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int h = 0;
    if (cudaMemcpyAsync(&h, st->status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return LQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return LQ_ERR_CUDA;
    if (h & lq::kStatusTimeout) return LQ_ERR_TIMEOUT;
    if (h & lq::kStatusNonFinite) return LQ_ERR_NONFINITE;
    return LQ_OK;
}

void lq_state_destroy(lq_state *st) {
    if (st) release(st);
}

const char *lq_strerror(int status) {
    switch (status) {
        case LQ_OK: return "ok";
        case LQ_ERR_INVALID_ARG: return "invalid argument";
        case LQ_ERR_SHAPE: return "inconsistent shape";
        case LQ_ERR_WORKSPACE: return "workspace too small or misaligned";
        case LQ_ERR_WINDOW_FULL: return "window full: flush before decoding another token";
        case LQ_ERR_CUDA: return "CUDA runtime error";
        case LQ_ERR_NONFINITE: return "non-finite value produced on the device";
        case LQ_ERR_UNSUPPORTED: return "unsupported head size or configuration";
        case LQ_ERR_TIMEOUT: return "a bounded device wait timed out";
        default: return "unknown status";
    }
}

}  // extern "C"
