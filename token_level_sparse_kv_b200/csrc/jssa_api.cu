// C ABI of libjssa (declared in include/jssa.h): host-side argument checks,
// workspace layout and kernel launches.  No allocation, no synchronisation.
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "jssa_internal.h"

namespace jssa {

cudaError_t ensure_smem(const void *kern, size_t smem) {
    if (smem <= 48 * 1024) return cudaSuccess;
    struct Entry {
        const void *kern;
        int dev;
        size_t smem;
    };
    static Entry table[256];
    static int n = 0;
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < n; ++i)
        if (table[i].kern == kern && table[i].dev == dev) {
            if (table[i].smem >= smem) return cudaSuccess;
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e == cudaSuccess) table[i].smem = smem;
            return e;
        }
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess && n < 256) table[n++] = Entry{kern, dev, smem};
    return e;
}

int device_sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        dev = 0;
    }
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = 1;
        }
        cache[dev] = n;
    }
    return cache[dev];
}

}  // namespace jssa

using namespace jssa;

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    cudaGetLastError();  // clear this runtime's last-error slot
    return fail(JSSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Shape {
    bool latent;
    int G, es_kv, es_kt;
    int BH;
};

int check_dims(const jssa_dims *d, Shape *sh) {
    if (!d) return fail(JSSA_ERR_INVALID_ARG, "dims is NULL");
    if (d->B < 0 || d->Hq < 1 || d->Hkv < 1 || d->T_cap < 1 || d->d < 1 || d->dv < 1 || d->r < 1)
        return fail(JSSA_ERR_INVALID_ARG, "bad dimension (B=%d Hq=%d Hkv=%d d=%d dv=%d r=%d T_cap=%d)", d->B, d->Hq,
                    d->Hkv, d->d, d->dv, d->r, d->T_cap);
    if (d->Hq % d->Hkv != 0) return fail(JSSA_ERR_INVALID_ARG, "Hq=%d is not a multiple of Hkv=%d", d->Hq, d->Hkv);
    if ((long long)d->B * d->Hkv > 65535) return fail(JSSA_ERR_UNSUPPORTED, "B*Hkv above 65535");
    if ((d->kv_dtype != JSSA_BF16 && d->kv_dtype != JSSA_FP32) || (d->kt_dtype != JSSA_BF16 && d->kt_dtype != JSSA_FP32))
        return fail(JSSA_ERR_INVALID_ARG, "bad dtype code (kv=%d kt=%d)", d->kv_dtype, d->kt_dtype);
    if (d->r > d->d) return fail(JSSA_ERR_INVALID_ARG, "r=%d exceeds d=%d", d->r, d->d);
    if (d->r < 8 || d->r > 128 || (d->r & (d->r - 1)) != 0)
        return fail(JSSA_ERR_UNSUPPORTED, "r=%d: supported ranks are powers of two in [8, 128]", d->r);
    const bool latent = d->d == 576 && d->dv == 512 && d->Hkv == 1;
    const bool gqa = (d->d == 64 || d->d == 128 || d->d == 256) && d->dv == d->d;
    if (!latent && !gqa)
        return fail(JSSA_ERR_UNSUPPORTED, "d=%d dv=%d: supported are d in {64,128,256} with dv=d, or d=576 dv=512 Hkv=1",
                    d->d, d->dv);
    sh->latent = latent;
    sh->G = d->Hq / d->Hkv;
    sh->es_kv = d->kv_dtype == JSSA_BF16 ? 2 : 4;
    sh->es_kt = d->kt_dtype == JSSA_BF16 ? 2 : 4;
    sh->BH = d->B * d->Hkv;
    return JSSA_OK;
}

// One selection (and attention) row per query head: the dims seen by the
// row-wise planners (Hkv = Hq rows, G = 1).
void heads_view(const jssa_dims *d, const Shape &sh, jssa_dims *dh, Shape *shh) {
    *dh = *d;
    dh->Hkv = d->Hq;
    *shh = sh;
    shh->G = 1;
    shh->BH = d->B * d->Hq;
}

int check_k(int k) {
    if (k < 1 || k > kMaxK) return fail(JSSA_ERR_INVALID_ARG, "k=%d outside [1, %d]", k, kMaxK);
    return JSSA_OK;
}

// Attention kernels exist for GQA (G <= 16, bf16 or fp32) and for the latent
// cache with 128 heads in bf16.
int check_attn_shape(const jssa_dims *d, const Shape &sh, bool indexed) {
    (void)indexed;
    if (sh.latent) {
        if (d->Hq != 128 || d->kv_dtype != JSSA_BF16)
            return fail(JSSA_ERR_UNSUPPORTED, "latent-cache attention needs Hq = 128 and bf16 (got Hq=%d)", d->Hq);
        return JSSA_OK;
    }
    if (sh.G > kMaxG) return fail(JSSA_ERR_UNSUPPORTED, "G=%d query heads per KV head above %d", sh.G, kMaxG);
    return JSSA_OK;
}

// The per-query-head variant: GQA shapes, G <= 16 (the per-head projection).
int check_heads_shape(const jssa_dims *d, const Shape &sh) {
    if (sh.latent) return fail(JSSA_ERR_UNSUPPORTED, "per-query-head selection is for GQA shapes, not the latent form");
    if (sh.G > kMaxG) return fail(JSSA_ERR_UNSUPPORTED, "per-query-head selection needs G <= %d (got %d)", kMaxG, sh.G);
    (void)d;
    return JSSA_OK;
}

#define REQUIRE_PTR(p)                                                                          \
    do {                                                                                        \
        if (!(p)) return fail(JSSA_ERR_INVALID_ARG, "%s is NULL", #p);                          \
        if (!aligned16(p)) return fail(JSSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p); \
    } while (0)
#define OPTIONAL_PTR(p)                                                                         \
    do {                                                                                        \
        if ((p) && !aligned16(p)) return fail(JSSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p); \
    } while (0)

// ----------------------------------------------------------- workspace ---
struct Layout {
    size_t qproj = 0, cand_key = 0, cand_idx = 0, cand_cnt = 0, sel_ctr = 0;
    size_t part_o = 0, part_ml = 0, att_ctr = 0, gcount = 0;
    size_t cal_sk = 0, cal_sq = 0, cal_m = 0;
    int cal_chunks = 0;
    size_t total = 256;  // [0, 256): status word
    ScanPlan sp{};
    AttnPlan ap{};
    bool csel = false;   // selection by one cluster per (b,h)
    bool wspec = false;  // warp-specialised streaming selection (else block-synchronous)
    bool fused = false;  // decode step in one launch of the streaming kernel
    ScanPlan fp{};
    CSelPlan cp{};
    bool tc = false;     // dense pass on the tensor cores (bf16)
    DensePlan dp{};
    MlaRangePlan mp{};   // latent cache, dense or gathered rows
};

size_t take(size_t &off, size_t bytes) {
    const size_t o = off;
    off = (off + bytes + 255) / 256 * 256;
    return o;
}

// Selection form: the cluster form where one wave of clusters covers the
// rows, else the streaming form, else the block-synchronous scan.  With
// stream_first (a decode step that runs as one fused launch of the streaming
// kernel) the streaming form is tried first.  A forced form (form != 0,
// jssa_select_form) overrides the choice.
int layout_select(const jssa_dims *d, const Shape &sh, int src, int k, int agg, int form, Layout &L,
                  bool stream_first = false, bool no_stream = false) {
    const int nq = (src != SRC_SCORES && agg == JSSA_AGG_MAX) ? sh.G : 1;
    stream_first = stream_first && form == JSSA_FORM_AUTO;
    auto try_csel = [&](bool &ok) -> int {
        ok = false;
        cudaError_t ec = plan_csel(form, src, agg, d->B, d->Hkv, d->T_cap, d->r, nq, k, &L.cp);
        if (ec == cudaSuccess) {
            L.csel = true;
            ok = true;
            return JSSA_OK;
        }
        cudaGetLastError();
        if (ec != cudaErrorNotSupported) return cuda_fail(ec, "planning the cluster selection");
        return JSSA_OK;
    };
    bool done = false;
    if (!stream_first) {
        const int st = try_csel(done);
        if (st != JSSA_OK || done) return st;
    }
    cudaError_t e = (form == JSSA_FORM_SCAN || no_stream) ? cudaErrorNotSupported : plan_stream(src, agg, d->B, d->Hkv, d->T_cap, d->r, k, &L.sp);
    if (e == cudaSuccess) {
        L.wspec = true;
    } else {
        cudaGetLastError();
        if (e != cudaErrorNotSupported) return cuda_fail(e, "planning the streaming selection");
        if (stream_first) {
            const int st = try_csel(done);
            if (st != JSSA_OK || done) return st;
        }
        e = plan_scan(src, MODE_SELECT, agg, d->B, d->Hkv, d->T_cap, d->r, nq, k, &L.sp);
        if (e != cudaSuccess) return cuda_fail(e, "planning the selection pass");
    }
    const size_t nc = (size_t)sh.BH * L.sp.max_seg * k;
    L.cand_key = take(L.total, nc * 4);
    L.cand_idx = take(L.total, nc * 4);
    L.cand_cnt = take(L.total, (size_t)sh.BH * L.sp.max_seg * 4);
    L.sel_ctr = take(L.total, (size_t)sh.BH * 2 * 4);  // tickets and publish counts
    return JSSA_OK;
}

int layout_attend(const jssa_dims *d, const Shape &sh, int src, int npos, Layout &L) {
    if (sh.latent && src != ATT_INDEXED) {
        cudaError_t e = plan_mla_range(d->B, npos, &L.mp);
        if (e != cudaSuccess) return cuda_fail(e, "planning the latent-cache range pass");
        L.part_o = take(L.total, (size_t)d->B * L.mp.splits * d->Hq * d->dv * 2);  // bf16
        L.part_ml = take(L.total, (size_t)d->B * L.mp.splits * d->Hq * 2 * 4);
        L.att_ctr = take(L.total, (size_t)sh.BH * 4);
        return JSSA_OK;
    }
    if (sh.latent) {
        L.ap = AttnPlan();
        L.ap.splits = mla_splits(npos);
        L.part_o = take(L.total, (size_t)d->B * L.ap.splits * d->Hq * d->dv * 2);  // bf16
        L.part_ml = take(L.total, (size_t)d->B * L.ap.splits * d->Hq * 2 * 4);
        L.att_ctr = take(L.total, (size_t)sh.BH * 2 * 4);  // arrival and done counters of the split merge
        return JSSA_OK;
    }
    if (src != ATT_INDEXED && d->kv_dtype == JSSA_BF16) {
        cudaError_t e = plan_dense(d->d, d->B, d->Hkv, npos, &L.dp);
        if (e == cudaSuccess) {
            L.tc = true;
            L.part_o = take(L.total, (size_t)sh.BH * L.dp.part_stride * sh.G * d->dv * 4);
            L.part_ml = take(L.total, (size_t)sh.BH * L.dp.part_stride * sh.G * 2 * 4);
            L.att_ctr = take(L.total, (size_t)sh.BH * 4);
            return JSSA_OK;
        }
        cudaGetLastError();
        if (e != cudaErrorNotSupported) return cuda_fail(e, "planning the dense pass");
    }
    cudaError_t e = plan_attend(src, d->kv_dtype, d->d, sh.G, d->B, d->Hkv, npos, &L.ap);
    if (e != cudaSuccess) return cuda_fail(e, "planning the attention pass");
    L.part_o = take(L.total, (size_t)sh.BH * L.ap.splits * sh.G * d->dv * 4);
    L.part_ml = take(L.total, (size_t)sh.BH * L.ap.splits * sh.G * 2 * 4);
    L.att_ctr = take(L.total, (size_t)sh.BH * 4);
    return JSSA_OK;
}

// Planning choices a caller can force (jssa_select_opts): the selection
// form, and whether the decode step may run as one fused launch.
struct Choice {
    int form = JSSA_FORM_AUTO;
    int unfused = 0;
};
Choice choice_of(const jssa_select_opts *opts) {
    Choice c;
    if (opts) {
        c.form = opts->form;
        c.unfused = opts->unfused ? 1 : 0;
    }
    return c;
}

int build_layout_uncached(const jssa_dims *d, const Shape &sh, int k, int op, int agg, int window, Choice ch,
                          Layout &L);

// Layouts (workspace offsets and kernel plans) are cached per device, dims,
// op and settings: planning costs occupancy queries and attribute calls that
// would otherwise dominate the host time of a decode step.  The kernels'
// shared-memory attributes set by the first planning stay set for the
// process, so a cached plan can be launched directly.
struct LayoutKey {
    int dev, op, k, agg, window, form, fused;
    jssa_dims dims;
    bool operator==(const LayoutKey &o) const { return !memcmp(this, &o, sizeof *this); }
};
struct LayoutEntry {
    LayoutKey key;
    Layout L;
};
constexpr int kLayoutCache = 64;
LayoutEntry g_layouts[kLayoutCache];
int g_layouts_n = 0, g_layouts_next = 0;
std::mutex g_layouts_mu;

int build_layout(const jssa_dims *d, const Shape &sh, int k, int op, int agg, int window, Choice ch, Layout &L) {
    LayoutKey key;
    memset(&key, 0, sizeof key);
    cudaError_t e = cudaGetDevice(&key.dev);
    if (e != cudaSuccess) return cuda_fail(e, "querying the current device");
    key.op = op;
    key.k = k;
    key.agg = agg;
    key.window = window;
    key.form = ch.form;
    key.fused = ch.unfused ? 0 : 1;
    key.dims = *d;
    {
        std::lock_guard<std::mutex> lk(g_layouts_mu);
        for (int i = 0; i < g_layouts_n; ++i)
            if (g_layouts[i].key == key) {
                L = g_layouts[i].L;
                return JSSA_OK;
            }
    }
    const int st = build_layout_uncached(d, sh, k, op, agg, window, ch, L);
    if (st != JSSA_OK) return st;
    std::lock_guard<std::mutex> lk(g_layouts_mu);
    LayoutEntry &slot = g_layouts[g_layouts_n < kLayoutCache ? g_layouts_n++ : (g_layouts_next++ % kLayoutCache)];
    slot.key = key;
    slot.L = L;
    return JSSA_OK;
}

int build_layout_uncached(const jssa_dims *d, const Shape &sh, int k, int op, int agg, int window, Choice ch,
                          Layout &L) {
    L = Layout();
    int st = JSSA_OK;
    const int nq = agg == JSSA_AGG_MAX ? sh.G : 1;
    switch (op) {
        case JSSA_OP_APPEND: break;
        case JSSA_OP_SCORE: {
            L.qproj = take(L.total, (size_t)sh.BH * nq * d->r * 4);
            cudaError_t e = plan_scan(d->kt_dtype == JSSA_BF16 ? SRC_KT_BF16 : SRC_KT_FP32, MODE_WRITE, agg, d->B,
                                      d->Hkv, d->T_cap, d->r, nq, 0, &L.sp);
            if (e != cudaSuccess) return cuda_fail(e, "planning the score pass");
            break;
        }
        case JSSA_OP_TOPK: st = layout_select(d, sh, SRC_SCORES, k, agg, ch.form, L); break;
        case JSSA_OP_SELECT:
            L.qproj = take(L.total, (size_t)sh.BH * nq * d->r * 4);
            st = layout_select(d, sh, d->kt_dtype == JSSA_BF16 ? SRC_KT_BF16 : SRC_KT_FP32, k, agg, ch.form, L);
            break;
        case JSSA_OP_INDEXED_DECODE: st = layout_attend(d, sh, ATT_INDEXED, k, L); break;
        case JSSA_OP_DENSE_DECODE:
            st = layout_attend(d, sh, ATT_RANGE, window > 0 && window < d->T_cap ? window : d->T_cap, L);
            break;
        case JSSA_OP_GATHER_THEN_DENSE:
            st = layout_attend(d, sh, ATT_RANGE_BH, k, L);
            if (st == JSSA_OK) L.gcount = take(L.total, (size_t)sh.BH * 4);
            break;
        case JSSA_OP_CALIBRATE: {
            const size_t dd = (size_t)d->d * d->d;
            L.cal_chunks = calib_chunks(d->Hkv);
            L.cal_sk = take(L.total, (size_t)d->Hkv * L.cal_chunks * dd * 4);
            L.cal_sq = take(L.total, (size_t)d->Hkv * dd * 4);
            L.cal_m = take(L.total, (size_t)d->Hkv * dd * 4);
            break;
        }
        case JSSA_OP_SELECT_HEADS: {
            L.qproj = take(L.total, (size_t)sh.BH * sh.G * d->r * 4);  // per-head projections
            jssa_dims dh;
            Shape shh;
            heads_view(d, sh, &dh, &shh);
            st = layout_select(&dh, shh, d->kt_dtype == JSSA_BF16 ? SRC_KT_BF16 : SRC_KT_FP32, k, JSSA_AGG_SUM,
                               ch.form == JSSA_FORM_STREAM ? JSSA_FORM_AUTO : ch.form, L, false, true);
            break;
        }
        case JSSA_OP_INDEXED_DECODE_HEADS: {
            jssa_dims dh;
            Shape shh;
            heads_view(d, sh, &dh, &shh);
            st = layout_attend(&dh, shh, ATT_INDEXED, k, L);
            break;
        }
        case JSSA_OP_DECODE_STEP: {
            // one fused launch where the shape allows it; with k <= 256 it
            // also beats the three-launch cluster form on short caches and
            // small batches, so the streaming form is then tried first (with a
            // larger k the cluster form keeps its place where it plans)
            ScanPlan fp{};
            bool fused_ok = false;
            if (!sh.latent && agg == JSSA_AGG_SUM && d->kv_dtype == JSSA_BF16 && d->kt_dtype == JSSA_BF16 &&
                !ch.unfused) {
                cudaError_t e = plan_step_fused(d->B, d->Hkv, d->Hq, d->d, d->T_cap, d->r, k, &fp);
                if (e == cudaSuccess) {
                    fused_ok = true;
                } else {
                    cudaGetLastError();
                    if (e != cudaErrorNotSupported) return cuda_fail(e, "planning the fused step");
                }
            }
            L.qproj = take(L.total, (size_t)sh.BH * nq * d->r * 4);
            st = layout_select(d, sh, d->kt_dtype == JSSA_BF16 ? SRC_KT_BF16 : SRC_KT_FP32, k, agg, ch.form, L,
                               fused_ok && k <= 256);
            if (st == JSSA_OK) st = layout_attend(d, sh, ATT_INDEXED, k, L);
            if (st == JSSA_OK && fused_ok && L.wspec && fp.max_seg <= L.sp.max_seg) {
                L.fp = fp;
                L.fused = true;
            }
            break;
        }
        default: return fail(JSSA_ERR_INVALID_ARG, "unknown op %d", op);
    }
    return st;
}

int check_ws(void *ws, size_t ws_bytes, const Layout &L) {
    if (!ws) return fail(JSSA_ERR_INVALID_ARG, "ws is NULL");
    if (!aligned16(ws)) return fail(JSSA_ERR_INVALID_ARG, "ws is not 16-byte aligned");
    if (ws_bytes < L.total)
        return fail(JSSA_ERR_WORKSPACE, "workspace of %zu bytes is below the %zu bytes needed", ws_bytes, L.total);
    return JSSA_OK;
}

template <typename T>
T *at(void *ws, size_t off) {
    return reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}

cudaStream_t S(jssa_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// Screening fields of a streaming-form launch (opts->block_norms non-null).
void fill_screen(ScanArgs &sa, const jssa_dims *d, const jssa_select_opts *opts, void *ws) {
    if (!opts || !opts->block_norms) return;
    sa.norms = opts->block_norms;
    sa.norm_blocks = (d->T_cap + JSSA_NORM_BLOCK - 1) / JSSA_NORM_BLOCK;
    sa.skip_count = at<uint32_t>(ws, 4);
}

int check_opts(const jssa_select_opts *opts) {
    if (!opts) return JSSA_OK;
    if (opts->n_sink < 0 || opts->n_recent < 0)
        return fail(JSSA_ERR_INVALID_ARG, "negative forced-token count (n_sink=%d, n_recent=%d)", opts->n_sink,
                    opts->n_recent);
    if (opts->form < JSSA_FORM_AUTO || opts->form > JSSA_FORM_SCAN)
        return fail(JSSA_ERR_INVALID_ARG, "unknown selection form %d", opts->form);
    if (opts->unfused != 0 && opts->unfused != 1)
        return fail(JSSA_ERR_INVALID_ARG, "unfused=%d is neither 0 nor 1", opts->unfused);
    if (opts->block_norms && !aligned16(opts->block_norms))
        return fail(JSSA_ERR_INVALID_ARG, "block_norms is not 16-byte aligned");
    return JSSA_OK;
}

void fill_attn(AttnArgs &a, const jssa_dims *d, const Shape &sh, const void *q, const void *K, const void *V,
               const int32_t *seq_lens, float scale, void *out, float *lse, void *ws, const Layout &L) {
    memset(&a, 0, sizeof a);
    a.q = q;
    a.K = K;
    a.V = V;
    a.k_sb = (long long)d->T_cap * d->Hkv * d->d;
    a.k_st = (long long)d->Hkv * d->d;
    a.k_sh = d->d;
    a.v_sb = (long long)d->T_cap * d->Hkv * d->dv;
    a.v_st = (long long)d->Hkv * d->dv;
    a.v_sh = d->dv;
    a.seq_lens = seq_lens;
    a.B = d->B;
    a.Hq = d->Hq;
    a.Hkv = d->Hkv;
    a.G = sh.G;
    a.T_cap = d->T_cap;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.part_o = at<float>(ws, L.part_o);
    a.part_ml = at<float>(ws, L.part_ml);
    a.counters = at<uint32_t>(ws, L.att_ctr);
    a.out = out;
    a.lse = lse;
    a.status = at<uint32_t>(ws, 0);
}

void fill_dense(DenseArgs &a, const jssa_dims *d, const Shape &sh, const void *q, const int32_t *seq_lens,
                float scale, void *out, float *lse, void *ws, const Layout &L) {
    memset(&a, 0, sizeof a);
    a.q = q;
    a.seq_lens = seq_lens;
    a.B = d->B;
    a.Hq = d->Hq;
    a.Hkv = d->Hkv;
    a.G = sh.G;
    a.T_cap = d->T_cap;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.part_o = at<float>(ws, L.part_o);
    a.part_ml = at<float>(ws, L.part_ml);
    a.counters = at<uint32_t>(ws, L.att_ctr);
    a.out = out;
    a.lse = lse;
    a.status = at<uint32_t>(ws, 0);
}

int run_select(const jssa_dims *d, const Shape &sh, const void *q, const float *P, const void *Kt,
               const int32_t *seq_lens, int agg, int k, int32_t *idx, int32_t *count, void *ws, const Layout &L,
               cudaStream_t s, bool with_project, const jssa_select_opts *opts, int src_div = 1) {
    const int n_sink = opts ? opts->n_sink : 0, n_recent = opts ? opts->n_recent : 0;
    const int nq = agg == JSSA_AGG_MAX ? sh.G : 1;
    if (with_project) {
        ProjArgs pj{q, P, at<float>(ws, L.qproj), d->B, d->Hq, d->Hkv, d->d, d->r, agg};
        cudaError_t e = launch_project(pj, s, true, d->kv_dtype);
        if (e != cudaSuccess) return cuda_fail(e, "launching the query projection");
    }
    if (L.csel) {
        CSelArgs ca;
        memset(&ca, 0, sizeof ca);
        ca.src = Kt;
        ca.qproj = at<float>(ws, L.qproj);
        ca.seq_lens = seq_lens;
        ca.idx_out = idx;
        ca.count_out = count;
        ca.status = at<uint32_t>(ws, 0);
        ca.B = d->B;
        ca.Hkv = d->Hkv;
        ca.T_cap = d->T_cap;
        ca.r = d->r;
        ca.nq = nq;
        ca.k = k;
        ca.n_sink = n_sink;
        ca.n_recent = n_recent;
        ca.src_div = src_div;
        // a null query means the source is a score array (jssa_topk)
        const int src = q == nullptr ? SRC_SCORES : (d->kt_dtype == JSSA_BF16 ? SRC_KT_BF16 : SRC_KT_FP32);
        cudaError_t e = launch_csel(L.cp, ca, src, q == nullptr ? JSSA_AGG_SUM : agg, s, true);
        if (e != cudaSuccess) return cuda_fail(e, "launching the cluster selection");
        return JSSA_OK;
    }
    ScanArgs sa;
    memset(&sa, 0, sizeof sa);
    sa.src = Kt;
    sa.qproj = at<float>(ws, L.qproj);
    sa.seq_lens = seq_lens;
    sa.cand_key = at<uint32_t>(ws, L.cand_key);
    sa.cand_idx = at<int32_t>(ws, L.cand_idx);
    sa.cand_cnt = at<int32_t>(ws, L.cand_cnt);
    sa.counters = at<uint32_t>(ws, L.sel_ctr);
    sa.idx_out = idx;
    sa.count_out = count;
    sa.status = at<uint32_t>(ws, 0);
    sa.B = d->B;
    sa.Hkv = d->Hkv;
    sa.T_cap = d->T_cap;
    sa.r = d->r;
    sa.nq = nq;
    sa.k = k;
    sa.n_sink = n_sink;
    sa.n_recent = n_recent;
    sa.src_div = src_div;
    if (L.wspec && q != nullptr && src_div <= 1) fill_screen(sa, d, opts, ws);
    cudaError_t e = L.wspec ? launch_stream(L.sp, sa, s, true) : launch_scan(L.sp, sa, agg, s, true);
    if (e != cudaSuccess) return cuda_fail(e, "launching the selection pass");
    return JSSA_OK;
}

int run_mla_range(const jssa_dims *d, const void *q, const void *K, const int32_t *seq_lens, const int32_t *count,
                  int k, float scale, void *out, float *lse, void *ws, const Layout &L, cudaStream_t s) {
    MlaRangeArgs a;
    memset(&a, 0, sizeof a);
    a.q = q;
    a.seq_lens = seq_lens;
    a.count = count;
    a.B = d->B;
    a.T_cap = d->T_cap;
    a.k = k;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.part_o = at<__nv_bfloat16>(ws, L.part_o);
    a.part_ml = at<float>(ws, L.part_ml);
    a.out = out;
    a.lse = lse;
    a.status = at<uint32_t>(ws, 0);
    cudaError_t e = launch_mla_range(L.mp, a, K, s, true);
    if (e != cudaSuccess) return cuda_fail(e, "launching the latent-cache range pass");
    return JSSA_OK;
}

int run_mla(const jssa_dims *d, const void *q, const void *K, const int32_t *idx, const int32_t *count, int k,
            const int32_t *seq_lens, float scale, void *out, float *lse, void *ws, const Layout &L, cudaStream_t s) {
    MlaArgs a;
    memset(&a, 0, sizeof a);
    a.q = q;
    a.K = K;
    a.idx = idx;
    a.count = count;
    a.seq_lens = seq_lens;
    a.k = k;
    a.T_cap = d->T_cap;
    a.B = d->B;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.splits = L.ap.splits;
    a.part_o = at<__nv_bfloat16>(ws, L.part_o);
    a.part_ml = at<float>(ws, L.part_ml);
    a.out = out;
    a.lse = lse;
    a.status = at<uint32_t>(ws, 0);
    a.ctr = at<uint32_t>(ws, L.att_ctr);
    cudaError_t e = launch_mla(a, true, s, true);
    if (e != cudaSuccess) return cuda_fail(e, "launching the latent-cache indexed decode");
    return JSSA_OK;
}

}  // namespace

extern "C" {

int jssa_version(void) { return JSSA_VERSION; }

const char *jssa_status_string(int status) {
    switch (status) {
        case JSSA_OK: return "JSSA_OK";
        case JSSA_ERR_INVALID_ARG: return "JSSA_ERR_INVALID_ARG: invalid argument";
        case JSSA_ERR_UNSUPPORTED: return "JSSA_ERR_UNSUPPORTED: shape or dtype without a kernel";
        case JSSA_ERR_WORKSPACE: return "JSSA_ERR_WORKSPACE: workspace too small";
        case JSSA_ERR_CUDA: return "JSSA_ERR_CUDA: CUDA runtime error";
        default: return "unknown status";
    }
}

const char *jssa_last_error(void) { return g_err; }

int jssa_workspace_size(const jssa_dims *dims, int k, int op, size_t *bytes) {
    Shape sh;
    int st = check_dims(dims, &sh);
    if (st) return st;
    if (!bytes) return fail(JSSA_ERR_INVALID_ARG, "bytes is NULL");
    const bool needs_k = op == JSSA_OP_TOPK || op == JSSA_OP_SELECT || op == JSSA_OP_INDEXED_DECODE ||
                         op == JSSA_OP_GATHER_THEN_DENSE || op == JSSA_OP_DECODE_STEP || op == JSSA_OP_SELECT_HEADS ||
                         op == JSSA_OP_INDEXED_DECODE_HEADS;
    if (needs_k && (st = check_k(k))) return st;
    if ((op == JSSA_OP_SELECT_HEADS || op == JSSA_OP_INDEXED_DECODE_HEADS) && (st = check_heads_shape(dims, sh)))
        return st;
    if ((op == JSSA_OP_INDEXED_DECODE || op == JSSA_OP_DENSE_DECODE || op == JSSA_OP_GATHER_THEN_DENSE ||
         op == JSSA_OP_DECODE_STEP) &&
        (st = check_attn_shape(dims, sh, op == JSSA_OP_INDEXED_DECODE || op == JSSA_OP_DECODE_STEP)))
        return st;
    const bool selects = op == JSSA_OP_TOPK || op == JSSA_OP_SELECT || op == JSSA_OP_DECODE_STEP ||
                         op == JSSA_OP_SELECT_HEADS;
    size_t best = 0;
    for (int agg = 0; agg < 2; ++agg) {
        if (agg == JSSA_AGG_MAX && sh.G > kMaxG) continue;
        for (int form = 0; form < (selects ? 4 : 1); ++form)
            for (int unf = 0; unf < (op == JSSA_OP_DECODE_STEP ? 2 : 1); ++unf) {
                Choice ch;
                ch.form = form;
                ch.unfused = unf;
                Layout L;
                st = build_layout(dims, sh, k, op, agg, 0, ch, L);
                if (st) return st;
                if (L.total > best) best = L.total;
            }
    }
    *bytes = best;
    return JSSA_OK;
}

int jssa_plan_info(const jssa_dims *dims, int k, int op, int agg, int *launches, char *desc, size_t desc_len) {
    return jssa_plan_info_ex(dims, k, op, agg, nullptr, launches, desc, desc_len);
}

int jssa_plan_info_ex(const jssa_dims *dims, int k, int op, int agg, const jssa_select_opts *opts, int *launches,
                      char *desc, size_t desc_len) {
    Shape sh;
    int st = check_dims(dims, &sh);
    if (st) return st;
    if (!launches) return fail(JSSA_ERR_INVALID_ARG, "launches is NULL");
    if (agg != JSSA_AGG_SUM && agg != JSSA_AGG_MAX) return fail(JSSA_ERR_INVALID_ARG, "bad agg %d", agg);
    const bool needs_k = op == JSSA_OP_TOPK || op == JSSA_OP_SELECT || op == JSSA_OP_INDEXED_DECODE ||
                         op == JSSA_OP_GATHER_THEN_DENSE || op == JSSA_OP_DECODE_STEP || op == JSSA_OP_SELECT_HEADS ||
                         op == JSSA_OP_INDEXED_DECODE_HEADS;
    if (needs_k && (st = check_k(k))) return st;
    if ((op == JSSA_OP_SELECT_HEADS || op == JSSA_OP_INDEXED_DECODE_HEADS) && (st = check_heads_shape(dims, sh)))
        return st;
    if ((st = check_opts(opts))) return st;
    Layout L;
    if ((st = build_layout(dims, sh, k, op, agg, 0, choice_of(opts), L))) return st;
    const char *sel = L.csel ? "cluster" : (L.wspec ? "stream" : "scan");
    const int att = sh.latent ? 1 + (L.ap.splits > 1 && !mla_inline_combine(L.ap.splits, dims->B) ? 1 : 0) : 1;
    int n = 0;
    char text[160];
    switch (op) {
        case JSSA_OP_APPEND: n = 1; snprintf(text, sizeof text, "append"); break;
        case JSSA_OP_SCORE: n = 2; snprintf(text, sizeof text, "projection + score pass"); break;
        case JSSA_OP_TOPK: n = 1; snprintf(text, sizeof text, "top-k (%s form)", sel); break;
        case JSSA_OP_SELECT: n = 2; snprintf(text, sizeof text, "projection + selection (%s form)", sel); break;
        case JSSA_OP_INDEXED_DECODE: n = att; snprintf(text, sizeof text, "indexed attention"); break;
        case JSSA_OP_SELECT_HEADS:
            n = 2;
            snprintf(text, sizeof text, "per-head projection + per-query-head selection (%s form)", sel);
            break;
        case JSSA_OP_INDEXED_DECODE_HEADS: n = 1; snprintf(text, sizeof text, "per-query-head indexed attention"); break;
        case JSSA_OP_DENSE_DECODE:
        case JSSA_OP_GATHER_THEN_DENSE: {
            const int g = op == JSSA_OP_GATHER_THEN_DENSE ? 1 : 0;
            if (sh.latent) {
                n = g + 1 + (L.mp.splits > 1 ? 1 : 0);
                snprintf(text, sizeof text, "%slatent-cache range attention (tensor cores)%s", g ? "gather + " : "",
                         L.mp.splits > 1 ? " + combine" : "");
            } else if (L.tc) {
                n = g + 2;
                snprintf(text, sizeof text, "%sdense attention (tensor cores) + combine", g ? "gather + " : "");
            } else {
                n = g + 1;
                snprintf(text, sizeof text, "%sdense attention", g ? "gather + " : "");
            }
            break;
        }
        case JSSA_OP_DECODE_STEP:
            if (L.fused) {
                n = 1;
                snprintf(text, sizeof text, "fused step (stream form: append, projection, selection, attention)");
            } else {
                n = 2 + att;
                snprintf(text, sizeof text, "append + projection, selection (%s form), attention", sel);
            }
            break;
        default: return fail(JSSA_ERR_INVALID_ARG, "unknown op %d", op);
    }
    *launches = n;
    if (desc && desc_len) {
        strncpy(desc, text, desc_len - 1);
        desc[desc_len - 1] = 0;
    }
    return JSSA_OK;
}

int jssa_workspace_init(void *ws, size_t ws_bytes, jssa_stream_t stream) {
    if (!ws) return fail(JSSA_ERR_INVALID_ARG, "ws is NULL");
    cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, S(stream));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the workspace");
    return JSSA_OK;
}

int jssa_append_lowrank(const jssa_dims *dims, const void *K, const float *P, void *Kt, const int32_t *pos_begin,
                        int n_new, void *ws, size_t ws_bytes, jssa_stream_t stream) {
    Shape sh;
    int st = check_dims(dims, &sh);
    if (st) return st;
    REQUIRE_PTR(K);
    REQUIRE_PTR(P);
    REQUIRE_PTR(Kt);
    REQUIRE_PTR(pos_begin);
    if (n_new < 0 || n_new > dims->T_cap) return fail(JSSA_ERR_INVALID_ARG, "n_new=%d outside [0, T_cap]", n_new);
    Layout L;
    if ((st = build_layout(dims, sh, 1, JSSA_OP_APPEND, 0, 0, Choice(), L))) return st;
    if ((st = check_ws(ws, ws_bytes, L))) return st;
    if (n_new == 0 || dims->B == 0) return JSSA_OK;
    AppendArgs a{K, P, Kt, pos_begin, at<uint32_t>(ws, 0), dims->B, dims->T_cap, dims->Hkv, dims->d, dims->r, n_new, 0};
    cudaError_t e = launch_append(a, S(stream), true, dims->kv_dtype, dims->kt_dtype);
    if (e != cudaSuccess) return cuda_fail(e, "launching the low-rank append");
    return JSSA_OK;
}

int jssa_score(const jssa_dims *dims, const void *q, const float *P, const void *Kt, const int32_t *seq_lens,
               int agg, float *scores, void *ws, size_t ws_bytes, jssa_stream_t stream) {
    Shape sh;
    int st = check_dims(dims, &sh);
    if (st) return st;
    REQUIRE_PTR(q);
    REQUIRE_PTR(P);
    REQUIRE_PTR(Kt);
    REQUIRE_PTR(seq_lens);
    REQUIRE_PTR(scores);
    if (agg != JSSA_AGG_SUM && agg != JSSA_AGG_MAX) return fail(JSSA_ERR_INVALID_ARG, "bad agg %d", agg);
    if (agg == JSSA_AGG_MAX && sh.G > kMaxG) return fail(JSSA_ERR_UNSUPPORTED, "MAX aggregation needs G <= %d", kMaxG);
    Layout L;
    if ((st = build_layout(dims, sh, 1, JSSA_OP_SCORE, agg, 0, Choice(), L))) return st;
    if ((st = check_ws(ws, ws_bytes, L))) return st;
    if (dims->B == 0) return JSSA_OK;
    const int nq = agg == JSSA_AGG_MAX ? sh.G : 1;
    ProjArgs pj{q, P, at<float>(ws, L.qproj), dims->B, dims->Hq, dims->Hkv, dims->d, dims->r, agg};
    cudaError_t e = launch_project(pj, S(stream), true, dims->kv_dtype);
    if (e != cudaSuccess) return cuda_fail(e, "launching the query projection");
    ScanArgs sa;
    memset(&sa, 0, sizeof sa);
    sa.src = Kt;
    sa.qproj = at<float>(ws, L.qproj);
    sa.seq_lens = seq_lens;
    sa.scores_out = scores;
    sa.status = at<uint32_t>(ws, 0);
    sa.B = dims->B;
    sa.Hkv = dims->Hkv;
    sa.T_cap = dims->T_cap;
    sa.r = dims->r;
    sa.nq = nq;
    e = launch_scan(L.sp, sa, agg, S(stream), true);
    if (e != cudaSuccess) return cuda_fail(e, "launching the score pass");
    return JSSA_OK;
}

int jssa_topk(const jssa_dims *dims, const float *scores, const int32_t *seq_lens, int k, int32_t *idx,
              int32_t *count, void *ws, size_t ws_bytes, jssa_stream_t stream) {
    return jssa_topk_ex(dims, scores, seq_lens, k, nullptr, idx, count, ws, ws_bytes, stream);
}

int jssa_topk_ex(const jssa_dims *dims, const float *scores, const int32_t *seq_lens, int k,
                 const jssa_select_opts *opts, int32_t *idx, int32_t *count, void *ws, size_t ws_bytes,
                 jssa_stream_t stream) {
    Shape sh;
    int st = check_dims(dims, &sh);
    if (st) return st;
    if ((st = check_k(k))) return st;
    REQUIRE_PTR(scores);
    REQUIRE_PTR(seq_lens);
    REQUIRE_PTR(idx);
    OPTIONAL_PTR(count);
    if ((st = check_opts(opts))) return st;
    Layout L;
    if ((st = build_layout(dims, sh, k, JSSA_OP_TOPK, 0, 0, choice_of(opts), L))) return st;
    if ((st = check_ws(ws, ws_bytes, L))) return st;
    if (dims->B == 0) return JSSA_OK;
    return run_select(dims, sh, nullptr, nullptr, scores, seq_lens, JSSA_AGG_SUM, k, idx, count, ws, L, S(stream),
                      false, opts);
}

int jssa_select(const jssa_dims *dims, const void *q, const float *P, const void *Kt, const int32_t *seq_lens,
                int agg, int k, int32_t *idx, int32_t *count, void *ws, size_t ws_bytes, jssa_stream_t stream) {
    return jssa_select_ex(dims, q, P, Kt, seq_lens, agg, k, nullptr, idx, count, ws, ws_bytes, stream);
}

int jssa_select_ex(const jssa_dims *dims, const void *q, const float *P, const void *Kt, const int32_t *seq_lens,
                   int agg, int k, const jssa_select_opts *opts, int32_t *idx, int32_t *count, void *ws,
                   size_t ws_bytes, jssa_stream_t stream) {
    Shape sh;
    int st = check_dims(dims, &sh);
    if (st) return st;
    if ((st = check_k(k))) return st;
    REQUIRE_PTR(q);
    REQUIRE_PTR(P);
    REQUIRE_PTR(Kt);
    REQUIRE_PTR(seq_lens);
    REQUIRE_PTR(idx);
    OPTIONAL_PTR(count);
    if (agg != JSSA_AGG_SUM && agg != JSSA_AGG_MAX) return fail(JSSA_ERR_INVALID_ARG, "bad agg %d", agg);
    if (agg == JSSA_AGG_MAX && sh.G > kMaxG) return fail(JSSA_ERR_UNSUPPORTED, "MAX aggregation needs G <= %d", kMaxG);
    if ((st = check_opts(opts))) return st;
    Layout L;
    if ((st = build_layout(dims, sh, k, JSSA_OP_SELECT, agg, 0, choice_of(opts), L))) return st;
    if ((st = check_ws(ws, ws_bytes, L))) return st;
    if (dims->B == 0) return JSSA_OK;
    return run_select(dims, sh, q, P, Kt, seq_lens, agg, k, idx, count, ws, L, S(stream), true, opts);
}

int jssa_indexed_decode(const jssa_dims *dims, const void *q, const void *K, const void *V, const int32_t *idx,
                        const int32_t *count, int k, const int32_t *seq_lens, float softmax_scale, void *out,
                        float *lse, void *ws, size_t ws_bytes, jssa_stream_t stream) {
    Shape sh;
    int st = check_dims(dims, &sh);
    if (st) return st;
    if ((st = check_k(k))) return st;
    if ((st = check_attn_shape(dims, sh, true))) return st;
    REQUIRE_PTR(q);
    REQUIRE_PTR(K);
    REQUIRE_PTR(V);
    REQUIRE_PTR(idx);
    REQUIRE_PTR(seq_lens);
    REQUIRE_PTR(out);
    OPTIONAL_PTR(count);
    OPTIONAL_PTR(lse);
    Layout L;
    if ((st = build_layout(dims, sh, k, JSSA_OP_INDEXED_DECODE, 0, 0, Choice(), L))) return st;
    if ((st = check_ws(ws, ws_bytes, L))) return st;
    if (dims->B == 0) return JSSA_OK;
    if (sh.latent) return run_mla(dims, q, K, idx, count, k, seq_lens, softmax_scale, out, lse, ws, L, S(stream));
    AttnArgs a;
    fill_attn(a, dims, sh, q, K, V, seq_lens, softmax_scale, out, lse, ws, L);
    a.idx = idx;
    a.count = count;
    a.k = k;
    cudaError_t e = launch_attend(L.ap, ATT_INDEXED, a, dims->kv_dtype, dims->d, S(stream), true);
    if (e != cudaSuccess) return cuda_fail(e, "launching the indexed decode");
    return JSSA_OK;
}

int jssa_dense_decode(const jssa_dims *dims, const void *q, const void *K, const void *V, const int32_t *seq_lens,
                      int window, float softmax_scale, void *out, float *lse, void *ws, size_t ws_bytes,
                      jssa_stream_t stream) {
    Shape sh;
    int st = check_dims(dims, &sh);
    if (st) return st;
    if ((st = check_attn_shape(dims, sh, false))) return st;
    if (window < 0) return fail(JSSA_ERR_INVALID_ARG, "window=%d is negative", window);
    if (sh.latent && window > 0 && window < dims->T_cap)
        return fail(JSSA_ERR_UNSUPPORTED, "sliding-window attention over a latent cache has no kernel in this library");
    REQUIRE_PTR(q);
    REQUIRE_PTR(K);
    REQUIRE_PTR(V);
    REQUIRE_PTR(seq_lens);
    REQUIRE_PTR(out);
    OPTIONAL_PTR(lse);
    Layout L;
    if ((st = build_layout(dims, sh, 1, JSSA_OP_DENSE_DECODE, 0, window, Choice(), L))) return st;
    if ((st = check_ws(ws, ws_bytes, L))) return st;
    if (dims->B == 0) return JSSA_OK;
    if (sh.latent)
        return run_mla_range(dims, q, K, seq_lens, nullptr, 0, softmax_scale, out, lse, ws, L, S(stream));
    if (L.tc) {
        DenseArgs da;
        fill_dense(da, dims, sh, q, seq_lens, softmax_scale, out, lse, ws, L);
        da.window = window;
        cudaError_t e = launch_dense(L.dp, da, K, V, dims->d, S(stream), true);
        if (e != cudaSuccess) return cuda_fail(e, "launching the dense decode");
        return JSSA_OK;
    }
    AttnArgs a;
    fill_attn(a, dims, sh, q, K, V, seq_lens, softmax_scale, out, lse, ws, L);
    a.window = window;
    cudaError_t e = launch_attend(L.ap, ATT_RANGE, a, dims->kv_dtype, dims->d, S(stream), true);
    if (e != cudaSuccess) return cuda_fail(e, "launching the dense decode");
    return JSSA_OK;
}

int jssa_gather_then_dense(const jssa_dims *dims, const void *q, const void *K, const void *V, const int32_t *idx,
                           const int32_t *count, int k, const int32_t *seq_lens, float softmax_scale,
                           void *gather_buf, size_t gather_bytes, void *out, float *lse, void *ws, size_t ws_bytes,
                           jssa_stream_t stream) {
    Shape sh;
    int st = check_dims(dims, &sh);
    if (st) return st;
    if ((st = check_k(k))) return st;
    if ((st = check_attn_shape(dims, sh, false))) return st;
    REQUIRE_PTR(q);
    REQUIRE_PTR(K);
    REQUIRE_PTR(V);
    REQUIRE_PTR(idx);
    REQUIRE_PTR(seq_lens);
    REQUIRE_PTR(out);
    REQUIRE_PTR(gather_buf);
    OPTIONAL_PTR(count);
    OPTIONAL_PTR(lse);
    const size_t half = (size_t)sh.BH * k * dims->d * sh.es_kv;
    const size_t need = sh.latent ? half : 2 * half;  // a latent row is its own value
    if (gather_bytes < need)
        return fail(JSSA_ERR_INVALID_ARG, "gather_buf of %zu bytes is below the %zu bytes needed", gather_bytes,
                    need);
    Layout L;
    if ((st = build_layout(dims, sh, k, JSSA_OP_GATHER_THEN_DENSE, 0, 0, Choice(), L))) return st;
    if ((st = check_ws(ws, ws_bytes, L))) return st;
    if (dims->B == 0) return JSSA_OK;
    void *gK = gather_buf;
    void *gV = sh.latent ? nullptr : static_cast<char *>(gather_buf) + half;
    GatherArgs g{K, sh.latent ? nullptr : V, idx, count, seq_lens, gK, gV, at<int32_t>(ws, L.gcount),
                 at<uint32_t>(ws, 0), dims->B, dims->Hkv, dims->T_cap, dims->d, k};
    cudaError_t e = launch_gather(g, dims->kv_dtype, S(stream), true);
    if (e != cudaSuccess) return cuda_fail(e, "launching the gather");
    if (sh.latent)
        return run_mla_range(dims, q, gK, seq_lens, at<int32_t>(ws, L.gcount), k, softmax_scale, out, lse, ws, L,
                             S(stream));
    if (L.tc) {
        DenseArgs da;
        fill_dense(da, dims, sh, q, seq_lens, softmax_scale, out, lse, ws, L);
        da.count = at<int32_t>(ws, L.gcount);
        da.k = k;
        e = launch_dense(L.dp, da, gK, gV, dims->d, S(stream), true);
        if (e != cudaSuccess) return cuda_fail(e, "launching the dense decode over gathered rows");
        return JSSA_OK;
    }
    AttnArgs a;
    fill_attn(a, dims, sh, q, gK, gV, seq_lens, softmax_scale, out, lse, ws, L);
    a.k_sb = a.v_sb = (long long)dims->Hkv * k * dims->d;
    a.k_st = a.v_st = dims->d;
    a.k_sh = a.v_sh = (long long)k * dims->d;
    a.count = at<int32_t>(ws, L.gcount);
    a.k = k;
    e = launch_attend(L.ap, ATT_RANGE_BH, a, dims->kv_dtype, dims->d, S(stream), true);
    if (e != cudaSuccess) return cuda_fail(e, "launching the dense decode over gathered rows");
    return JSSA_OK;
}

int jssa_decode_step(const jssa_dims *dims, const void *q, const void *K, const void *V, const float *P, void *Kt,
                     const int32_t *seq_lens, const int32_t *pos_begin, int k, int agg, float softmax_scale,
                     int32_t *idx, int32_t *count, void *out, float *lse, void *ws, size_t ws_bytes,
                     jssa_stream_t stream) {
    return jssa_decode_step_ex(dims, q, K, V, P, Kt, seq_lens, pos_begin, k, agg, softmax_scale, nullptr, idx, count,
                               out, lse, ws, ws_bytes, stream);
}

int jssa_decode_step_ex(const jssa_dims *dims, const void *q, const void *K, const void *V, const float *P,
                        void *Kt, const int32_t *seq_lens, const int32_t *pos_begin, int k, int agg,
                        float softmax_scale, const jssa_select_opts *opts, int32_t *idx, int32_t *count, void *out,
                        float *lse, void *ws, size_t ws_bytes, jssa_stream_t stream) {
    Shape sh;
    int st = check_dims(dims, &sh);
    if (st) return st;
    if ((st = check_k(k))) return st;
    if ((st = check_attn_shape(dims, sh, true))) return st;
    REQUIRE_PTR(q);
    REQUIRE_PTR(K);
    REQUIRE_PTR(V);
    REQUIRE_PTR(P);
    REQUIRE_PTR(Kt);
    REQUIRE_PTR(seq_lens);
    REQUIRE_PTR(pos_begin);
    REQUIRE_PTR(idx);
    REQUIRE_PTR(count);
    REQUIRE_PTR(out);
    OPTIONAL_PTR(lse);
    if (agg != JSSA_AGG_SUM && agg != JSSA_AGG_MAX) return fail(JSSA_ERR_INVALID_ARG, "bad agg %d", agg);
    if ((st = check_opts(opts))) return st;
    Layout L;
    if ((st = build_layout(dims, sh, k, JSSA_OP_DECODE_STEP, agg, 0, choice_of(opts), L))) return st;
    if ((st = check_ws(ws, ws_bytes, L))) return st;
    if (dims->B == 0) return JSSA_OK;
    if (L.fused) {
        ScanArgs sa;
        memset(&sa, 0, sizeof sa);
        sa.src = Kt;
        sa.seq_lens = seq_lens;
        sa.cand_key = at<uint32_t>(ws, L.cand_key);
        sa.cand_idx = at<int32_t>(ws, L.cand_idx);
        sa.cand_cnt = at<int32_t>(ws, L.cand_cnt);
        sa.counters = at<uint32_t>(ws, L.sel_ctr);
        sa.idx_out = idx;
        sa.count_out = count;
        sa.status = at<uint32_t>(ws, 0);
        sa.B = dims->B;
        sa.Hkv = dims->Hkv;
        sa.T_cap = dims->T_cap;
        sa.r = dims->r;
        sa.nq = 1;
        sa.k = k;
        sa.n_sink = opts ? opts->n_sink : 0;
        sa.n_recent = opts ? opts->n_recent : 0;
        fill_screen(sa, dims, opts, ws);
        StepExtra x;
        x.q = q;
        x.P = P;
        x.K = K;
        x.V = V;
        x.pos_begin = pos_begin;
        x.out = out;
        x.lse = lse;
        x.scale_log2 = softmax_scale * 1.4426950408889634f;
        x.Hq = dims->Hq;
        x.G = sh.G;
        x.d = dims->d;
        cudaError_t e = launch_step_fused(L.fp, sa, x, S(stream), true);
        if (e != cudaSuccess) return cuda_fail(e, "launching the fused decode step");
        return JSSA_OK;
    }
    AppendArgs ap{K, P, Kt, pos_begin, at<uint32_t>(ws, 0), dims->B, dims->T_cap, dims->Hkv, dims->d, dims->r, 1, 1};
    ProjArgs pj{q, P, at<float>(ws, L.qproj), dims->B, dims->Hq, dims->Hkv, dims->d, dims->r, agg};
    cudaError_t e = launch_prep(ap, pj, S(stream), true, dims->kv_dtype, dims->kt_dtype);
    if (e != cudaSuccess) return cuda_fail(e, "launching the append + projection prologue");
    if (opts && opts->block_norms && !sh.latent) {
        e = launch_norm_raise(Kt, dims->kt_dtype, opts->block_norms, pos_begin, dims->B, dims->Hkv, dims->T_cap,
                              dims->r, S(stream), true);
        if (e != cudaSuccess) return cuda_fail(e, "launching the screening-bound update");
    }
    if ((st = run_select(dims, sh, q, P, Kt, seq_lens, agg, k, idx, count, ws, L, S(stream), false, opts)))
        return st;
    if (sh.latent) return run_mla(dims, q, K, idx, count, k, seq_lens, softmax_scale, out, lse, ws, L, S(stream));
    AttnArgs a;
    fill_attn(a, dims, sh, q, K, V, seq_lens, softmax_scale, out, lse, ws, L);
    a.idx = idx;
    a.count = count;
    a.k = k;
    e = launch_attend(L.ap, ATT_INDEXED, a, dims->kv_dtype, dims->d, S(stream), true);
    if (e != cudaSuccess) return cuda_fail(e, "launching the indexed decode");
    return JSSA_OK;
}

int jssa_block_norms(const jssa_dims *dims, const void *Kt, float *norms, jssa_stream_t stream) {
    // only the low-rank cache's dims matter here: B, Hkv, T_cap, r, kt_dtype
    if (!dims) return fail(JSSA_ERR_INVALID_ARG, "dims is NULL");
    if (dims->B < 0 || dims->Hkv < 1 || dims->T_cap < 1 || dims->r < 1)
        return fail(JSSA_ERR_INVALID_ARG, "bad dimension (B=%d Hkv=%d r=%d T_cap=%d)", dims->B, dims->Hkv, dims->r,
                    dims->T_cap);
    if (dims->kt_dtype != JSSA_BF16 && dims->kt_dtype != JSSA_FP32)
        return fail(JSSA_ERR_INVALID_ARG, "bad dtype code (kt=%d)", dims->kt_dtype);
    if ((long long)dims->B * dims->Hkv > 65535) return fail(JSSA_ERR_UNSUPPORTED, "B*Hkv above 65535");
    REQUIRE_PTR(Kt);
    REQUIRE_PTR(norms);
    if (dims->B == 0) return JSSA_OK;
    cudaError_t e = launch_block_norms(Kt, dims->kt_dtype, norms, dims->B * dims->Hkv, dims->T_cap, dims->r,
                                       S(stream), true);
    if (e != cudaSuccess) return cuda_fail(e, "launching the block norms");
    return JSSA_OK;
}

int jssa_calibrate_basis(const jssa_dims *dims, const void *q_cal, int n_q, const void *K, const int32_t *seq_lens,
                         int n_keys, int iters, const float *P_init, float *P_out, void *ws, size_t ws_bytes,
                         jssa_stream_t stream) {
    Shape sh;
    int st = check_dims(dims, &sh);
    if (st) return st;
    if (sh.latent) return fail(JSSA_ERR_UNSUPPORTED, "calibration is for GQA shapes");
    if (dims->r > 64) return fail(JSSA_ERR_UNSUPPORTED, "calibration needs r <= 64 (got %d)", dims->r);
    if (n_q < 0 || n_keys < 0 || iters < 0 || iters > 1000)
        return fail(JSSA_ERR_INVALID_ARG, "bad counts (n_q=%d n_keys=%d iters=%d)", n_q, n_keys, iters);
    if (n_q > 0) REQUIRE_PTR(q_cal);
    REQUIRE_PTR(K);
    REQUIRE_PTR(seq_lens);
    REQUIRE_PTR(P_init);
    REQUIRE_PTR(P_out);
    if (P_init == P_out) return fail(JSSA_ERR_INVALID_ARG, "P_init and P_out alias");
    Layout L;
    if ((st = build_layout(dims, sh, 1, JSSA_OP_CALIBRATE, 0, 0, Choice(), L))) return st;
    if ((st = check_ws(ws, ws_bytes, L))) return st;
    CalibArgs a;
    memset(&a, 0, sizeof a);
    a.q = q_cal;
    a.K = K;
    a.seq_lens = seq_lens;
    a.B = dims->B;
    a.Hq = dims->Hq;
    a.Hkv = dims->Hkv;
    a.T_cap = dims->T_cap;
    a.Nq = n_q;
    a.n_keys = n_keys;
    a.chunks = L.cal_chunks;
    a.r = dims->r;
    a.iters = iters;
    a.P_init = P_init;
    a.P_out = P_out;
    a.Sk = at<float>(ws, L.cal_sk);
    a.Sq = at<float>(ws, L.cal_sq);
    a.M = at<float>(ws, L.cal_m);
    a.status = at<uint32_t>(ws, 0);
    cudaError_t e = launch_calib(a, dims->kv_dtype, dims->d, S(stream));
    if (e != cudaSuccess) return cuda_fail(e, "launching the calibration");
    return JSSA_OK;
}

int jssa_host_step_bytes(const jssa_dims *dims, size_t *bytes) {
    Shape sh;
    int st = check_dims(dims, &sh);
    if (st) return st;
    if (!bytes) return fail(JSSA_ERR_INVALID_ARG, "bytes is NULL");
    const size_t q = (size_t)dims->B * dims->Hq * dims->d, kr = (size_t)sh.BH * dims->d;
    const size_t vr = sh.latent ? 0 : (size_t)sh.BH * dims->dv;
    *bytes = (q + kr + vr) * sh.es_kv;
    return JSSA_OK;
}

int jssa_decode_step_host(const jssa_dims *dims, const void *in_host, void *stage, void *K, void *V, const float *P,
                          void *Kt, const int32_t *seq_lens, const int32_t *pos_begin, int k, int agg,
                          float softmax_scale, const jssa_select_opts *opts, int32_t *idx, int32_t *count, void *out,
                          float *lse, void *out_host, void *ws, size_t ws_bytes, jssa_stream_t stream) {
    Shape sh;
    int st = check_dims(dims, &sh);
    if (st) return st;
    if (!in_host) return fail(JSSA_ERR_INVALID_ARG, "in_host is NULL");
    if (!out_host) return fail(JSSA_ERR_INVALID_ARG, "out_host is NULL");
    REQUIRE_PTR(stage);
    REQUIRE_PTR(K);
    REQUIRE_PTR(V);
    size_t in_bytes = 0;
    if ((st = jssa_host_step_bytes(dims, &in_bytes))) return st;
    const size_t q_bytes = (size_t)dims->B * dims->Hq * dims->d * sh.es_kv;
    const size_t krow = (size_t)dims->Hkv * dims->d * sh.es_kv, vrow = (size_t)dims->Hkv * dims->dv * sh.es_kv;
    if (q_bytes % 16 || krow % 16 || vrow % 16)
        return fail(JSSA_ERR_UNSUPPORTED, "host-buffer step needs rows of whole 16-byte chunks");
    // argument checks of the step itself, before anything is enqueued
    {
        Layout L;
        if ((st = check_k(k))) return st;
        if ((st = check_attn_shape(dims, sh, true))) return st;
        if ((st = check_opts(opts))) return st;
        if (agg != JSSA_AGG_SUM && agg != JSSA_AGG_MAX) return fail(JSSA_ERR_INVALID_ARG, "bad agg %d", agg);
        if ((st = build_layout(dims, sh, k, JSSA_OP_DECODE_STEP, agg, 0, choice_of(opts), L))) return st;
        if ((st = check_ws(ws, ws_bytes, L))) return st;
    }
    if (dims->B == 0) return JSSA_OK;
    cudaError_t e = cudaMemcpyAsync(stage, in_host, in_bytes, cudaMemcpyHostToDevice, S(stream));
    if (e != cudaSuccess) return cuda_fail(e, "copying the step's inputs to the device");
    char *sg = static_cast<char *>(stage);
    const char *k_new = sg + q_bytes;
    const char *v_new = sh.latent ? nullptr : k_new + (size_t)dims->B * krow;
    e = launch_place_rows(k_new, v_new, K, sh.latent ? nullptr : V, pos_begin, dims->B, dims->T_cap, krow, vrow,
                          at<uint32_t>(ws, 0), S(stream), false);
    if (e != cudaSuccess) return cuda_fail(e, "launching the new-row write");
    st = jssa_decode_step_ex(dims, stage, K, V, P, Kt, seq_lens, pos_begin, k, agg, softmax_scale, opts, idx, count,
                             out, lse, ws, ws_bytes, stream);
    if (st) return st;
    e = cudaMemcpyAsync(out_host, out, (size_t)dims->B * dims->Hq * dims->dv * sh.es_kv, cudaMemcpyDeviceToHost,
                        S(stream));
    if (e != cudaSuccess) return cuda_fail(e, "copying the output to the host");
    return JSSA_OK;
}

int jssa_select_heads(const jssa_dims *dims, const void *q, const float *P, const void *Kt, const int32_t *seq_lens,
                      int k, const jssa_select_opts *opts, int32_t *idx, int32_t *count, void *ws, size_t ws_bytes,
                      jssa_stream_t stream) {
    Shape sh;
    int st = check_dims(dims, &sh);
    if (st) return st;
    if ((st = check_k(k))) return st;
    if ((st = check_heads_shape(dims, sh))) return st;
    REQUIRE_PTR(q);
    REQUIRE_PTR(P);
    REQUIRE_PTR(Kt);
    REQUIRE_PTR(seq_lens);
    REQUIRE_PTR(idx);
    OPTIONAL_PTR(count);
    if ((st = check_opts(opts))) return st;
    Layout L;
    if ((st = build_layout(dims, sh, k, JSSA_OP_SELECT_HEADS, 0, 0, choice_of(opts), L))) return st;
    if ((st = check_ws(ws, ws_bytes, L))) return st;
    if (dims->B == 0) return JSSA_OK;
    // per-head projections (the MAX layout: [B*Hkv, G, r] = one row per query head)
    ProjArgs pj{q, P, at<float>(ws, L.qproj), dims->B, dims->Hq, dims->Hkv, dims->d, dims->r, JSSA_AGG_MAX};
    cudaError_t e = launch_project(pj, S(stream), true, dims->kv_dtype);
    if (e != cudaSuccess) return cuda_fail(e, "launching the per-head projection");
    jssa_dims dh;
    Shape shh;
    heads_view(dims, sh, &dh, &shh);
    return run_select(&dh, shh, q, P, Kt, seq_lens, JSSA_AGG_SUM, k, idx, count, ws, L, S(stream), false, opts, sh.G);
}

int jssa_indexed_decode_heads(const jssa_dims *dims, const void *q, const void *K, const void *V, const int32_t *idx,
                              const int32_t *count, int k, const int32_t *seq_lens, float softmax_scale, void *out,
                              float *lse, void *ws, size_t ws_bytes, jssa_stream_t stream) {
    Shape sh;
    int st = check_dims(dims, &sh);
    if (st) return st;
    if ((st = check_k(k))) return st;
    if ((st = check_heads_shape(dims, sh))) return st;
    REQUIRE_PTR(q);
    REQUIRE_PTR(K);
    REQUIRE_PTR(V);
    REQUIRE_PTR(idx);
    REQUIRE_PTR(seq_lens);
    REQUIRE_PTR(out);
    OPTIONAL_PTR(count);
    OPTIONAL_PTR(lse);
    Layout L;
    if ((st = build_layout(dims, sh, k, JSSA_OP_INDEXED_DECODE_HEADS, 0, 0, Choice(), L))) return st;
    if ((st = check_ws(ws, ws_bytes, L))) return st;
    if (dims->B == 0) return JSSA_OK;
    AttnArgs a;
    fill_attn(a, dims, sh, q, K, V, seq_lens, softmax_scale, out, lse, ws, L);  // strides of the real cache
    a.Hkv = dims->Hq;  // one attention row per query head ...
    a.G = 1;
    a.head_div = sh.G;  // ... reading KV head g / G
    a.idx = idx;
    a.count = count;
    a.k = k;
    cudaError_t e = launch_attend(L.ap, ATT_INDEXED, a, dims->kv_dtype, dims->d, S(stream), true);
    if (e != cudaSuccess) return cuda_fail(e, "launching the per-query-head indexed decode");
    return JSSA_OK;
}

int jssa_check_wait_expiry(void *ws, size_t ws_bytes, uint64_t limit_ns, jssa_stream_t stream) {
    if (!ws) return fail(JSSA_ERR_INVALID_ARG, "ws is NULL");
    if (!aligned16(ws)) return fail(JSSA_ERR_INVALID_ARG, "ws is not 16-byte aligned");
    if (ws_bytes < 256) return fail(JSSA_ERR_WORKSPACE, "workspace of %zu bytes is below 256", ws_bytes);
    if (limit_ns < 1000 || limit_ns > 1000000000ull)
        return fail(JSSA_ERR_INVALID_ARG, "limit_ns=%llu outside [1000, 1e9]", (unsigned long long)limit_ns);
    cudaError_t e = cudaMemsetAsync(static_cast<char *>(ws) + 64, 0, 192, S(stream));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the self-check words");
    e = launch_wait_expiry(ws, limit_ns, S(stream));
    if (e != cudaSuccess) return cuda_fail(e, "launching the wait self-check");
    return JSSA_OK;
}

}  // extern "C"

// ------------------------------------------------------ allocation-free ---
// jssa_indexed_decode_noalloc: the indexed decode with its scratch (split
// partials, arrival counters, status word) in a fixed device array owned by
// the library instead of a caller workspace.  Each device that loads the
// library holds kNoAllocBytes of it until the process exits.
namespace {

constexpr size_t kNoAllocBytes = size_t(8) << 20;  // 8 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
void *g_noalloc_ptr[kMaxDevices] = {nullptr};
std::mutex g_noalloc_mu;

// Device address of the scratch array for the current device (looked up once
// per device, with that device current).  The cached address belongs to the
// device's primary context: after cudaDeviceReset() it is stale, and the
// library must be unloaded and loaded again before the next call.
int noalloc_scratch(void **ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "querying the current device");
    if (dev < 0 || dev >= kMaxDevices) return fail(JSSA_ERR_UNSUPPORTED, "device index %d above %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "looking up the allocation-free scratch array");
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    return JSSA_OK;
}

}  // namespace

extern "C" int jssa_indexed_decode_noalloc(const jssa_dims *dims, const void *q, const void *K, const void *V,
                                           const int32_t *idx, const int32_t *count, int k,
                                           const int32_t *seq_lens, float softmax_scale, void *out, float *lse,
                                           jssa_stream_t stream) {
    Shape sh;
    int st = check_dims(dims, &sh);
    if (st) return st;
    if ((st = check_k(k))) return st;
    if ((st = check_attn_shape(dims, sh, true))) return st;
    REQUIRE_PTR(q);
    REQUIRE_PTR(K);
    REQUIRE_PTR(V);
    REQUIRE_PTR(idx);
    REQUIRE_PTR(seq_lens);
    REQUIRE_PTR(out);
    OPTIONAL_PTR(count);
    OPTIONAL_PTR(lse);
    Layout L;
    if ((st = build_layout(dims, sh, k, JSSA_OP_INDEXED_DECODE, 0, 0, Choice(), L))) return st;
    if (L.total > kNoAllocBytes)
        return fail(JSSA_ERR_WORKSPACE,
                    "this shape needs %zu bytes of scratch, above the %zu bytes of the allocation-free entry point; "
                    "use jssa_indexed_decode with a caller workspace",
                    L.total, kNoAllocBytes);
    if (dims->B == 0) return JSSA_OK;
    void *ws = nullptr;
    if ((st = noalloc_scratch(&ws))) return st;
    // the status word and the arrival counters must start at zero
    cudaError_t e = cudaMemsetAsync(ws, 0, 256, S(stream));
    if (e == cudaSuccess)
        e = cudaMemsetAsync(at<char>(ws, L.att_ctr), 0, (size_t)sh.BH * 4 * (sh.latent ? 2 : 1), S(stream));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the allocation-free scratch");
    // the latent-cache form keeps its split partials in the same array (the
    // layout's offsets all lie below L.total, checked above)
    if (sh.latent) return run_mla(dims, q, K, idx, count, k, seq_lens, softmax_scale, out, lse, ws, L, S(stream));
    AttnArgs a;
    fill_attn(a, dims, sh, q, K, V, seq_lens, softmax_scale, out, lse, ws, L);
    a.idx = idx;
    a.count = count;
    a.k = k;
    e = launch_attend(L.ap, ATT_INDEXED, a, dims->kv_dtype, dims->d, S(stream), true);
    if (e != cudaSuccess) return cuda_fail(e, "launching the indexed decode");
    return JSSA_OK;
}
