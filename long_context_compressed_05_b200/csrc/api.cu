// C ABI entry points of libhcsa.so: argument validation on the host, then the
// kernel launches on the caller's stream.  See include/hca_csa.h for the
// contract of every call.
#include <stdio.h>

#include "internal.cuh"

namespace hcsa {

static __device__ int g_status_word;
static int *g_status_ptr[64];
static thread_local int64_t g_launches = 0;

int *device_status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = (int *)p;
    }
    return g_status_ptr[dev];
}

void count_launch(int n) { g_launches += n; }

hcsa_status check_launch() {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        fprintf(stderr, "hcsa: launch failed: %s\n", cudaGetErrorString(e));
        return HCSA_ERR_CUDA;
    }
    return HCSA_OK;
}

}  // namespace hcsa

using namespace hcsa;

namespace {

int esize(int dtype) { return dtype == HCSA_BF16 ? 2 : 4; }
int vec(int dtype) { return dtype == HCSA_BF16 ? 8 : 4; }
bool aligned(const void *p) { return ((uintptr_t)p & 15u) == 0; }
bool ld_ok(int dtype, int64_t ld, int64_t used) { return ld >= used && (ld * esize(dtype)) % 16 == 0; }

#define HCSA_TRY(expr)                       \
    do {                                     \
        hcsa_status _s = (expr);             \
        if (_s != HCSA_OK) return _s;        \
    } while (0)

hcsa_status check_common(const hcsa_params *p) {
    if (!p) return HCSA_ERR_NULL;
    if (p->dtype != HCSA_F32 && p->dtype != HCSA_BF16) return HCSA_ERR_DTYPE;
    const int V = vec(p->dtype);
    if (p->m < 1 || p->width < p->m || p->width > 512 || p->C < 2 || p->C % (2 * V) != 0) return HCSA_ERR_SHAPE;
    if (p->H < 1 || p->dh != p->C / 2 || p->window < 1) return HCSA_ERR_SHAPE;
    if (p->lowprec != 0 && p->lowprec != 1) return HCSA_ERR_SHAPE;
    if (p->lowprec && (p->dtype != HCSA_BF16 || p->C % 32 != 0)) return HCSA_ERR_UNSUPPORTED;
    return HCSA_OK;
}

hcsa_status check_csa(const hcsa_params *p) {
    HCSA_TRY(check_common(p));
    if (p->di < 1 || p->di > p->C || p->di % vec(p->dtype) != 0 || p->Hi < 1 || p->topk < 1)
        return HCSA_ERR_SHAPE;
    if (p->lowprec && p->di % 32 != 0) return HCSA_ERR_UNSUPPORTED;
    return HCSA_OK;
}

hcsa_status check_decode(const hcsa_params *p, const hcsa_cache *c, const int32_t *pos, bool csa) {
    if (!c || !pos || !c->entries || !c->win_kv || !c->ring_g) return HCSA_ERR_NULL;
    if (p->ent0 < 0 || (p->ent_shard != 0 && p->ent_shard != 1) || (!p->ent_shard && p->ent0 != 0))
        return HCSA_ERR_SHAPE;
    if (csa && (!c->idx_keys || !c->ring_ki)) return HCSA_ERR_NULL;
    if (p->B < 1 || p->n_cap < 1 || p->window < p->width) return HCSA_ERR_SHAPE;
    if (!aligned(c->entries) || !aligned(c->win_kv) || !aligned(c->ring_g) || !aligned(pos)) return HCSA_ERR_ALIGN;
    if (csa && (!aligned(c->idx_keys) || !aligned(c->ring_ki))) return HCSA_ERR_ALIGN;
    return HCSA_OK;
}

int64_t n_entries(const hcsa_params *p) { return ((int64_t)p->T + p->m - 1) / p->m; }

size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

// segment partials of a sharded decode attention (before their merge into the caller's partial)
size_t shard_part_ws(const hcsa_params *p, bool dense) {
    return attend_ws_bytes(HCSA_BF16, true, dense, p->B, p->H, p->dh, dense ? 0 : p->topk, p->window, p->n_cap);
}

// Prefill row range [r0, r1) of the T query rows (both fields 0: all rows).
hcsa_status row_range(const hcsa_params *p, int64_t *r0, int64_t *r1) {
    if (p->row0 == 0 && p->row1 == 0) {
        *r0 = 0;
        *r1 = p->T;
        return HCSA_OK;
    }
    if (p->row0 < 0 || p->row1 < p->row0 || p->row1 > p->T || p->row0 % 128 != 0 ||
        (p->row1 % 128 != 0 && p->row1 != p->T))
        return HCSA_ERR_SHAPE;
    *r0 = p->row0;
    *r1 = p->row1;
    return HCSA_OK;
}

// Entries whose pools end in rows [r0, r1): j in [r0 / m, ceil(r1 / m)) (r1 < T is a multiple of m).
void entry_range(const hcsa_params *p, int64_t r0, int64_t r1, int64_t *j0, int64_t *j1) {
    *j0 = r0 / p->m;
    *j1 = r1 == p->T ? n_entries(p) : r1 / p->m;
}

}  // namespace

namespace hcsa {

hcsa_status check_decode_index_topk_args(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos,
                                         const void *qi, int64_t ld_qi, const void *w, int64_t ld_w,
                                         const int32_t *sel) {
    HCSA_TRY(check_csa(p));
    HCSA_TRY(check_decode(p, cache, pos, true));
    if (!qi || !w || !sel) return HCSA_ERR_NULL;
    if (!aligned(qi) || !aligned(w) || !aligned(sel)) return HCSA_ERR_ALIGN;
    if (ld_qi < (int64_t)p->Hi * p->di || ld_w < p->Hi) return HCSA_ERR_SHAPE;
    return HCSA_OK;
}

}  // namespace hcsa

extern "C" {

int32_t hcsa_version(void) { return 100; }

const char *hcsa_status_string(hcsa_status s) {
    switch (s) {
        case HCSA_OK: return "ok";
        case HCSA_ERR_NULL: return "null pointer argument";
        case HCSA_ERR_SHAPE: return "invalid shape or size";
        case HCSA_ERR_DTYPE: return "unsupported storage dtype";
        case HCSA_ERR_ALIGN: return "pointer or leading dimension not 16-byte aligned";
        case HCSA_ERR_WORKSPACE: return "workspace too small";
        case HCSA_ERR_CUDA: return "CUDA launch or runtime error";
        case HCSA_ERR_TIMEOUT: return "a bounded device-side wait gave up";
        case HCSA_ERR_UNSUPPORTED: return "configuration not supported by the library";
        case HCSA_ERR_DEVICE: return "device-side bounds check failed";
    }
    return "unknown status";
}

int64_t hcsa_proj_cols(const hcsa_params *p, int32_t kind) {
    if (!p) return -1;
    int64_t c = 2 * (int64_t)p->C + (int64_t)p->H * p->dh;
    if (kind == HCSA_KIND_CSA) c += (int64_t)p->di + (int64_t)p->Hi * p->di + p->Hi;
    return c;
}

size_t hcsa_entry_bytes(const hcsa_params *p, int64_t rows) {
    if (!p || rows < 0) return 0;
    if (p->lowprec) return (size_t)rows * (p->C + p->C / 32);
    return (size_t)rows * p->C * esize(p->dtype);
}

size_t hcsa_key_bytes(const hcsa_params *p, int64_t rows) {
    if (!p || rows < 0) return 0;
    if (p->lowprec) return (size_t)rows * (p->di / 2 + p->di / 32);
    return (size_t)rows * p->di * esize(p->dtype);
}

size_t hcsa_workspace_bytes(const hcsa_params *p, int32_t op) {
    if (!p) return 0;
    switch (op) {
        case HCSA_OP_PROJECT: return project_ws_bytes(p->dtype);
        case HCSA_OP_CSA_INDEX_TOPK: return index_topk_ws_bytes(p->dtype, p->T, n_entries(p));
        case HCSA_OP_CSA_ATTEND: return attend_ws_bytes(p->dtype, false, false, p->T, p->H, p->dh, p->topk,
                                                        p->window, n_entries(p));
        case HCSA_OP_HCA_ATTEND: return attend_ws_bytes(p->dtype, false, true, p->T, p->H, p->dh, 0, p->window,
                                                        n_entries(p));
        case HCSA_OP_CSA_DECODE_INDEX_TOPK: {
            size_t b = index_topk_ws_bytes(p->dtype, p->B, p->n_cap);
            if (p->dtype == HCSA_BF16 && p->n_cap > 32768) b = ((b + 255) & ~(size_t)255) + topk_rows_ws_bytes(p->B);
            return b;
        }
        case HCSA_OP_CSA_DECODE_ATTEND: return attend_ws_bytes(p->dtype, true, false, p->B, p->H, p->dh, p->topk,
                                                               p->window, p->n_cap);
        case HCSA_OP_HCA_DECODE_ATTEND: return attend_ws_bytes(p->dtype, true, true, p->B, p->H, p->dh, 0,
                                                               p->window, p->n_cap);
        case HCSA_OP_CSA_DECODE_INDEX_TOPK_SHARD:
            return align256(hcsa_workspace_bytes(p, HCSA_OP_CSA_DECODE_INDEX_TOPK)) + (size_t)p->B * sizeof(int32_t);
        case HCSA_OP_CSA_DECODE_ATTEND_SHARD:
            return align256((size_t)p->B * p->topk * sizeof(int32_t)) + shard_part_ws(p, false);
        case HCSA_OP_HCA_DECODE_ATTEND_SHARD: return shard_part_ws(p, true);
    }
    return 0;
}

hcsa_status hcsa_project(const hcsa_params *p, int32_t kind, int64_t rows, const void *x, const void *W_cat,
                         void *y, void *ws, size_t ws_bytes, void *stream) {
    if (kind == HCSA_KIND_CSA) HCSA_TRY(check_csa(p));
    else if (kind == HCSA_KIND_HCA) HCSA_TRY(check_common(p));
    else return HCSA_ERR_SHAPE;
    if (!x || !W_cat || !y) return HCSA_ERR_NULL;
    if (rows < 0 || p->D < 1) return HCSA_ERR_SHAPE;
    if (!aligned(x) || !aligned(W_cat) || !aligned(y)) return HCSA_ERR_ALIGN;
    const int64_t nc = hcsa_proj_cols(p, kind);
    if ((p->D * esize(p->dtype)) % 16 || (nc * esize(p->dtype)) % 16) return HCSA_ERR_ALIGN;
    if (p->dtype == HCSA_BF16 && ws && ws_bytes < project_ws_bytes(p->dtype)) return HCSA_ERR_WORKSPACE;
    return launch_project(p->dtype, rows, p->D, nc, x, W_cat, y, ws, ws_bytes, (cudaStream_t)stream);
}

hcsa_status hcsa_out_project(const hcsa_params *p, int64_t rows, const void *out, int64_t ld_out, const void *W_o,
                             void *x, int64_t ld_x, void *ws, size_t ws_bytes, void *stream) {
    HCSA_TRY(check_common(p));
    if (p->dtype != HCSA_BF16) return HCSA_ERR_UNSUPPORTED;
    if (!out || !W_o || !x) return HCSA_ERR_NULL;
    if (rows < 0 || p->D < 1) return HCSA_ERR_SHAPE;
    if (p->T == 0 && rows > p->B) return HCSA_ERR_SHAPE;   // decode: one row per sequence of the batch
    const int64_t hd = (int64_t)p->H * p->dh;
    if (!aligned(out) || !aligned(W_o) || !aligned(x)) return HCSA_ERR_ALIGN;
    if (!ld_ok(p->dtype, ld_out, hd) || !ld_ok(p->dtype, ld_x, p->D) || (p->D * esize(p->dtype)) % 16)
        return HCSA_ERR_ALIGN;
    if (ws && ws_bytes < project_ws_bytes(p->dtype)) return HCSA_ERR_WORKSPACE;
    return launch_out_project(rows, hd, p->D, out, ld_out, W_o, x, ld_x, ws, ws_bytes, (cudaStream_t)stream);
}

hcsa_status csa_compress(const hcsa_params *p, const void *kv, int64_t ld_kv, const void *g, int64_t ld_g,
                         const void *ki, int64_t ld_ki, const void *bias, void *entries, void *idx_keys,
                         void *stream) {
    HCSA_TRY(check_csa(p));
    if (!kv || !g || !ki || !bias || !entries || !idx_keys) return HCSA_ERR_NULL;
    if (p->T < 0) return HCSA_ERR_SHAPE;
    if (!aligned(kv) || !aligned(g) || !aligned(ki) || !aligned(bias) || !aligned(entries) || !aligned(idx_keys))
        return HCSA_ERR_ALIGN;
    if (!ld_ok(p->dtype, ld_kv, p->C) || !ld_ok(p->dtype, ld_g, p->C) || !ld_ok(p->dtype, ld_ki, p->di))
        return HCSA_ERR_ALIGN;
    int64_t r0, r1, j0, j1;
    HCSA_TRY(row_range(p, &r0, &r1));
    entry_range(p, r0, r1, &j0, &j1);
    return launch_compress(p->dtype, p->T, p->C, p->m, p->width, kv, ld_kv, g, ld_g, ki, ld_ki, p->di, bias,
                           entries, idx_keys, j0, j1, p->lowprec != 0, n_entries(p), (cudaStream_t)stream);
}

hcsa_status hca_compress(const hcsa_params *p, const void *kv, int64_t ld_kv, const void *g, int64_t ld_g,
                         const void *bias, void *entries, void *stream) {
    HCSA_TRY(check_common(p));
    if (!kv || !g || !bias || !entries) return HCSA_ERR_NULL;
    if (p->T < 0) return HCSA_ERR_SHAPE;
    if (!aligned(kv) || !aligned(g) || !aligned(bias) || !aligned(entries)) return HCSA_ERR_ALIGN;
    if (!ld_ok(p->dtype, ld_kv, p->C) || !ld_ok(p->dtype, ld_g, p->C)) return HCSA_ERR_ALIGN;
    int64_t r0, r1, j0, j1;
    HCSA_TRY(row_range(p, &r0, &r1));
    entry_range(p, r0, r1, &j0, &j1);
    return launch_compress(p->dtype, p->T, p->C, p->m, p->width, kv, ld_kv, g, ld_g, nullptr, 0, 0, bias, entries,
                           nullptr, j0, j1, p->lowprec != 0, n_entries(p), (cudaStream_t)stream);
}

hcsa_status csa_index_topk(const hcsa_params *p, const void *qi, int64_t ld_qi, const void *w, int64_t ld_w,
                           const void *idx_keys, int32_t *sel, void *ws, size_t ws_bytes, void *stream) {
    HCSA_TRY(check_csa(p));
    if (!qi || !w || !idx_keys || !sel) return HCSA_ERR_NULL;
    if (p->T < 0) return HCSA_ERR_SHAPE;
    if (!aligned(qi) || !aligned(w) || !aligned(idx_keys) || !aligned(sel)) return HCSA_ERR_ALIGN;
    if (ld_qi < (int64_t)p->Hi * p->di || ld_w < p->Hi) return HCSA_ERR_SHAPE;
    if (!ws && p->T > 0) return HCSA_ERR_WORKSPACE;
    if (ws_bytes < hcsa_workspace_bytes(p, HCSA_OP_CSA_INDEX_TOPK)) return HCSA_ERR_WORKSPACE;
    int64_t r0, r1;
    HCSA_TRY(row_range(p, &r0, &r1));
    IndexArgs a{p->dtype, p->T, p->Hi, p->di, p->topk, p->m, n_entries(p), qi, ld_qi, w, ld_w, idx_keys,
                nullptr, sel, ws, ws_bytes, nullptr, r0, r1, p->lowprec != 0};
    return launch_index_topk(a, (cudaStream_t)stream);
}

static hcsa_status attend_prefill(const hcsa_params *p, bool dense, const void *q, int64_t ld_q, const void *kv,
                                  int64_t ld_kv, const void *entries, const int32_t *sel, void *out, void *ws,
                                  size_t ws_bytes, void *stream) {
    if (!q || !kv || !entries || !out || (!dense && !sel)) return HCSA_ERR_NULL;
    if (p->T < 0) return HCSA_ERR_SHAPE;
    if (!aligned(q) || !aligned(kv) || !aligned(entries) || !aligned(out)) return HCSA_ERR_ALIGN;
    if (ld_q < (int64_t)p->H * p->dh || ld_kv < p->C) return HCSA_ERR_SHAPE;
    int64_t r0, r1;
    HCSA_TRY(row_range(p, &r0, &r1));
    AttendArgs a{};
    a.dtype = p->dtype; a.rows = p->T; a.H = p->H; a.dh = p->dh; a.C = p->C; a.window = p->window; a.m = p->m;
    a.topk = dense ? 0 : p->topk; a.scale = p->scale; a.dense = dense; a.N = n_entries(p);
    a.row0 = r0; a.row1 = r1; a.lowprec = p->lowprec != 0;
    a.q = q; a.ld_q = ld_q; a.kv = kv; a.ld_kv = ld_kv; a.entries = entries; a.sel = sel; a.pos = nullptr;
    a.out = out; a.ws = ws; a.ws_bytes = ws_bytes;
    return launch_attend(a, (cudaStream_t)stream);
}

hcsa_status csa_attend(const hcsa_params *p, const void *q, int64_t ld_q, const void *kv, int64_t ld_kv,
                       const void *entries, const int32_t *sel, void *out, void *ws, size_t ws_bytes,
                       void *stream) {
    HCSA_TRY(check_csa(p));
    return attend_prefill(p, false, q, ld_q, kv, ld_kv, entries, sel, out, ws, ws_bytes, stream);
}

hcsa_status hca_attend(const hcsa_params *p, const void *q, int64_t ld_q, const void *kv, int64_t ld_kv,
                       const void *entries, void *out, void *ws, size_t ws_bytes, void *stream) {
    HCSA_TRY(check_common(p));
    if (p->lowprec) return HCSA_ERR_UNSUPPORTED;
    return attend_prefill(p, true, q, ld_q, kv, ld_kv, entries, nullptr, out, ws, ws_bytes, stream);
}

hcsa_status hcsa_cache_append(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos, const void *kv,
                              int64_t ld_kv, const void *g, int64_t ld_g, const void *ki, int64_t ld_ki,
                              const void *bias, void *stream) {
    const bool csa = ki != nullptr;
    HCSA_TRY(csa ? check_csa(p) : check_common(p));
    HCSA_TRY(check_decode(p, cache, pos, csa));
    if (!kv || !g || !bias) return HCSA_ERR_NULL;
    if (!aligned(kv) || !aligned(g) || !aligned(bias) || (csa && !aligned(ki))) return HCSA_ERR_ALIGN;
    if (!ld_ok(p->dtype, ld_kv, p->C) || !ld_ok(p->dtype, ld_g, p->C) || (csa && !ld_ok(p->dtype, ld_ki, p->di)))
        return HCSA_ERR_ALIGN;
    return launch_cache_append(p->dtype, *p, *cache, pos, kv, ld_kv, g, ld_g, ki, ld_ki, bias,
                               (cudaStream_t)stream);
}

hcsa_status hcsa_project_compress(const hcsa_params *p, int32_t kind, const void *x, const void *W_cat,
                                  const void *bias, void *y, void *entries, void *idx_keys, void *ws, size_t ws_bytes,
                                  void *stream) {
    const bool csa = kind == HCSA_KIND_CSA;
    if (kind != HCSA_KIND_CSA && kind != HCSA_KIND_HCA) return HCSA_ERR_SHAPE;
    HCSA_TRY(csa ? check_csa(p) : check_common(p));
    if (!x || !W_cat || !y || !bias || !entries || (csa && !idx_keys)) return HCSA_ERR_NULL;
    if (p->T < 0 || p->D < 1) return HCSA_ERR_SHAPE;
    if (!aligned(x) || !aligned(W_cat) || !aligned(y) || !aligned(bias) || !aligned(entries) ||
        (csa && !aligned(idx_keys)))
        return HCSA_ERR_ALIGN;
    const int64_t nc = hcsa_proj_cols(p, kind);
    if ((p->D * esize(p->dtype)) % 16 || (nc * esize(p->dtype)) % 16) return HCSA_ERR_ALIGN;
    int64_t r0, r1, j0, j1;
    HCSA_TRY(row_range(p, &r0, &r1));
    entry_range(p, r0, r1, &j0, &j1);
    cudaStream_t st = (cudaStream_t)stream;
    if (p->T == 0) return HCSA_OK;
    if (r0 == 0 && r1 == p->T && project_compress_supported(*p, csa))
        return launch_project_compress(*p, x, W_cat, nc, y, bias, entries, idx_keys, st);
    // other shapes and row ranges: the projection, then the compressor kernel
    if (p->dtype == HCSA_BF16 && ws && ws_bytes < project_ws_bytes(p->dtype)) return HCSA_ERR_WORKSPACE;
    HCSA_TRY(launch_project(p->dtype, p->T, p->D, nc, x, W_cat, y, ws, ws_bytes, st));
    const uint8_t *y8 = (const uint8_t *)y;
    const int es = esize(p->dtype);
    return launch_compress(p->dtype, p->T, p->C, p->m, p->width, y8, nc, y8 + (int64_t)p->C * es, nc,
                           csa ? y8 + 2 * (int64_t)p->C * es : nullptr, nc, csa ? p->di : 0, bias, entries,
                           csa ? idx_keys : nullptr, j0, j1, p->lowprec != 0, n_entries(p), st);
}

hcsa_status hcsa_project_append(const hcsa_params *p, int32_t kind, const hcsa_cache *cache, const int32_t *pos,
                                const void *x, const void *W_cat, const void *bias, void *y, void *ws, size_t ws_bytes,
                                void *stream) {
    const bool csa = kind == HCSA_KIND_CSA;
    if (kind != HCSA_KIND_CSA && kind != HCSA_KIND_HCA) return HCSA_ERR_SHAPE;
    HCSA_TRY(csa ? check_csa(p) : check_common(p));
    HCSA_TRY(check_decode(p, cache, pos, csa));
    if (!x || !W_cat || !y || !bias) return HCSA_ERR_NULL;
    if (p->D < 1) return HCSA_ERR_SHAPE;
    if (!aligned(x) || !aligned(W_cat) || !aligned(y) || !aligned(bias)) return HCSA_ERR_ALIGN;
    const int64_t nc = hcsa_proj_cols(p, kind);
    if ((p->D * esize(p->dtype)) % 16 || (nc * esize(p->dtype)) % 16) return HCSA_ERR_ALIGN;
    cudaStream_t st = (cudaStream_t)stream;
    if (project_append_supported(*p, csa))
        return launch_project_append(*p, csa, *cache, pos, x, W_cat, nc, y, bias, st);
    // other shapes: the projection, then the append kernel
    if (p->dtype == HCSA_BF16 && ws && ws_bytes < project_ws_bytes(p->dtype)) return HCSA_ERR_WORKSPACE;
    HCSA_TRY(launch_project(p->dtype, p->B, p->D, nc, x, W_cat, y, ws, ws_bytes, st));
    const int64_t ld = nc;
    const uint8_t *y8 = (const uint8_t *)y;
    const int es = esize(p->dtype);
    return launch_cache_append(p->dtype, *p, *cache, pos, y8, ld, y8 + (int64_t)p->C * es, ld,
                               csa ? y8 + 2 * (int64_t)p->C * es : nullptr, ld, bias, st);
}

hcsa_status csa_decode_index_topk(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos,
                                  const void *qi, int64_t ld_qi, const void *w, int64_t ld_w, int32_t *sel,
                                  void *ws, size_t ws_bytes, void *stream) {
    HCSA_TRY(hcsa::check_decode_index_topk_args(p, cache, pos, qi, ld_qi, w, ld_w, sel));
    if (!ws || ws_bytes < hcsa_workspace_bytes(p, HCSA_OP_CSA_DECODE_INDEX_TOPK)) return HCSA_ERR_WORKSPACE;
    IndexArgs a{p->dtype, p->B, p->Hi, p->di, p->topk, p->m, p->n_cap, qi, ld_qi, w, ld_w, cache->idx_keys,
                pos, sel, ws, ws_bytes, nullptr, 0, p->B, p->lowprec != 0};
    return launch_index_topk(a, (cudaStream_t)stream);
}

static hcsa_status attend_decode(const hcsa_params *p, bool dense, const hcsa_cache *cache, const int32_t *pos,
                                 const void *q, int64_t ld_q, const int32_t *sel, void *out, void *ws,
                                 size_t ws_bytes, void *stream) {
    if (!q || !out || (!dense && !sel)) return HCSA_ERR_NULL;
    if (!aligned(q) || !aligned(out)) return HCSA_ERR_ALIGN;
    if (ld_q < (int64_t)p->H * p->dh) return HCSA_ERR_SHAPE;
    const size_t need = hcsa_workspace_bytes(p, dense ? HCSA_OP_HCA_DECODE_ATTEND : HCSA_OP_CSA_DECODE_ATTEND);
    if (need && (!ws || ws_bytes < need)) return HCSA_ERR_WORKSPACE;
    AttendArgs a{};
    a.dtype = p->dtype; a.rows = p->B; a.H = p->H; a.dh = p->dh; a.C = p->C; a.window = p->window; a.m = p->m;
    a.topk = dense ? 0 : p->topk; a.scale = p->scale; a.dense = dense; a.N = p->n_cap;
    a.q = q; a.ld_q = ld_q; a.kv = cache->win_kv; a.ld_kv = p->C; a.entries = cache->entries; a.sel = sel;
    a.pos = pos; a.out = out; a.ws = ws; a.ws_bytes = ws_bytes;
    a.row0 = 0; a.row1 = p->B; a.lowprec = p->lowprec != 0;
    return launch_attend(a, (cudaStream_t)stream);
}

hcsa_status csa_decode_attend(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos, const void *q,
                              int64_t ld_q, const int32_t *sel, void *out, void *ws, size_t ws_bytes,
                              void *stream) {
    HCSA_TRY(check_csa(p));
    HCSA_TRY(check_decode(p, cache, pos, true));
    return attend_decode(p, false, cache, pos, q, ld_q, sel, out, ws, ws_bytes, stream);
}

hcsa_status hca_decode_attend(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos, const void *q,
                              int64_t ld_q, void *out, void *ws, size_t ws_bytes, void *stream) {
    HCSA_TRY(check_common(p));
    HCSA_TRY(check_decode(p, cache, pos, false));
    return attend_decode(p, true, cache, pos, q, ld_q, nullptr, out, ws, ws_bytes, stream);
}

hcsa_status hcsa_quantize_rows(const hcsa_params *p, int32_t what, const void *src, int64_t rows, void *dst,
                               void *stream) {
    if (!p) return HCSA_ERR_NULL;
    if (what != HCSA_STORE_ENTRIES && what != HCSA_STORE_KEYS) return HCSA_ERR_SHAPE;
    const bool keys = what == HCSA_STORE_KEYS;
    HCSA_TRY(keys ? check_csa(p) : check_common(p));
    if (!p->lowprec) return HCSA_ERR_UNSUPPORTED;
    if (!src || !dst) return HCSA_ERR_NULL;
    if (rows < 0) return HCSA_ERR_SHAPE;
    if (!aligned(src) || !aligned(dst)) return HCSA_ERR_ALIGN;
    return launch_quantize_rows(src, rows, keys ? p->di : p->C, keys, dst, (cudaStream_t)stream);
}

// ---------------------------------------------------------------- entry-sharded decode
static hcsa_status check_shard(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos, bool csa) {
    HCSA_TRY(csa ? check_csa(p) : check_common(p));
    HCSA_TRY(check_decode(p, cache, pos, csa));
    if (!p->ent_shard) return HCSA_ERR_SHAPE;
    if (p->dtype != HCSA_BF16 || p->lowprec) return HCSA_ERR_UNSUPPORTED;
    return HCSA_OK;
}

hcsa_status csa_decode_index_topk_shard(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos,
                                        const void *qi, int64_t ld_qi, const void *w, int64_t ld_w, int32_t *sel,
                                        float *sel_scores, void *ws, size_t ws_bytes, void *stream) {
    HCSA_TRY(check_shard(p, cache, pos, true));
    HCSA_TRY(hcsa::check_decode_index_topk_args(p, cache, pos, qi, ld_qi, w, ld_w, sel));
    if (!sel_scores) return HCSA_ERR_NULL;
    if (!aligned(sel_scores)) return HCSA_ERR_ALIGN;
    const size_t idx_ws = hcsa_workspace_bytes(p, HCSA_OP_CSA_DECODE_INDEX_TOPK);
    if (!ws || ws_bytes < hcsa_workspace_bytes(p, HCSA_OP_CSA_DECODE_INDEX_TOPK_SHARD)) return HCSA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    // the shard's entries are local rows 0 .. n_cap - 1: its visible count is that at position pos - m ent0
    int32_t *pos_l = reinterpret_cast<int32_t *>((uint8_t *)ws + align256(idx_ws));
    HCSA_TRY(launch_shift_pos(pos, p->B, (int64_t)p->m * p->ent0, pos_l, st));
    IndexArgs a{p->dtype, p->B, p->Hi, p->di, p->topk, p->m, p->n_cap, qi, ld_qi, w, ld_w, cache->idx_keys,
                pos_l, sel, ws, idx_ws, nullptr, 0, p->B, false};
    HCSA_TRY(launch_index_topk(a, st));
    return launch_shard_finish(sel, p->B, p->topk, (const float *)ws, p->n_cap, p->ent0, sel_scores, st);
}

hcsa_status csa_topk_merge(const hcsa_params *p, const int32_t *cand_sel, const float *cand_scores, int32_t n_cand,
                           int32_t *sel, void *stream) {
    if (!p) return HCSA_ERR_NULL;
    if (!cand_sel || !cand_scores || !sel) return HCSA_ERR_NULL;
    if (p->B < 1 || p->topk < 1) return HCSA_ERR_SHAPE;
    if (!topk_merge_supported(n_cand, p->topk)) return HCSA_ERR_UNSUPPORTED;
    return launch_topk_merge(cand_sel, cand_scores, p->B, n_cand, p->topk, sel, (cudaStream_t)stream);
}

static hcsa_status attend_shard(const hcsa_params *p, bool dense, const hcsa_cache *cache, const int32_t *pos,
                                const void *q, int64_t ld_q, const int32_t *sel, int32_t with_window, float *part,
                                void *ws, size_t ws_bytes, cudaStream_t st) {
    if (!q || !part || (!dense && !sel)) return HCSA_ERR_NULL;
    if (!aligned(q) || !aligned(part)) return HCSA_ERR_ALIGN;
    if (ld_q < (int64_t)p->H * p->dh) return HCSA_ERR_SHAPE;
    const size_t need = hcsa_workspace_bytes(p, dense ? HCSA_OP_HCA_DECODE_ATTEND_SHARD : HCSA_OP_CSA_DECODE_ATTEND_SHARD);
    if (need && (!ws || ws_bytes < need)) return HCSA_ERR_WORKSPACE;
    AttendArgs a{};
    a.dtype = p->dtype; a.rows = p->B; a.H = p->H; a.dh = p->dh; a.C = p->C; a.window = p->window; a.m = p->m;
    a.topk = dense ? 0 : p->topk; a.scale = p->scale; a.dense = dense; a.N = p->n_cap;
    a.q = q; a.ld_q = ld_q; a.kv = cache->win_kv; a.ld_kv = p->C; a.entries = cache->entries; a.pos = pos;
    a.row0 = 0; a.row1 = p->B; a.ent0 = p->ent0; a.no_window = with_window == 0;
    if (!attend_tc_supported(a)) return HCSA_ERR_UNSUPPORTED;
    uint8_t *w8 = (uint8_t *)ws;
    if (!dense) {   // the selection in the shard's local rows
        int32_t *sel_l = reinterpret_cast<int32_t *>(w8);
        HCSA_TRY(launch_localize_sel(sel, (int64_t)p->B * p->topk, p->ent0, p->n_cap, sel_l, st));
        a.sel = sel_l;
        w8 += align256((size_t)p->B * p->topk * sizeof(int32_t));
    }
    const int ns = attend_tc_segments(a);
    const int64_t nacc = (int64_t)p->B * p->H * p->dh;
    if (ns == 1) {   // one segment per row: the kernel writes the partial itself
        a.ws = part;
        a.ws_bytes = (size_t)(nacc + 2 * (int64_t)p->B * p->H) * sizeof(float);
        a.partial_out = true;
        return launch_attend_tc(a, st);
    }
    a.ws = w8;
    a.ws_bytes = shard_part_ws(p, dense);
    a.partial_out = true;
    HCSA_TRY(launch_attend_tc(a, st));
    const float *acc = (const float *)w8;
    const float *ml = acc + (int64_t)p->B * ns * p->H * p->dh;
    return launch_merge_parts(acc, ml, (int64_t)p->H * p->dh, (int64_t)ns * p->H * p->dh, p->H, (int64_t)ns * p->H,
                              ns, p->B, p->H, p->dh, nullptr, part, part + nacc, st);
}

hcsa_status csa_decode_attend_shard(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos, const void *q,
                                    int64_t ld_q, const int32_t *sel, int32_t with_window, float *part, void *ws,
                                    size_t ws_bytes, void *stream) {
    HCSA_TRY(check_shard(p, cache, pos, true));
    if (sel && !aligned(sel)) return HCSA_ERR_ALIGN;
    return attend_shard(p, false, cache, pos, q, ld_q, sel, with_window, part, ws, ws_bytes, (cudaStream_t)stream);
}

hcsa_status hca_decode_attend_shard(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos, const void *q,
                                    int64_t ld_q, int32_t with_window, float *part, void *ws, size_t ws_bytes,
                                    void *stream) {
    HCSA_TRY(check_shard(p, cache, pos, false));
    return attend_shard(p, true, cache, pos, q, ld_q, nullptr, with_window, part, ws, ws_bytes, (cudaStream_t)stream);
}

hcsa_status hcsa_merge_partials(const hcsa_params *p, const float *parts, int32_t n_parts, void *out, int64_t ld_out,
                                void *stream) {
    if (!p) return HCSA_ERR_NULL;
    if (!parts || !out) return HCSA_ERR_NULL;
    if (p->B < 1 || p->H < 1 || p->dh < 1 || n_parts < 1) return HCSA_ERR_SHAPE;
    if (ld_out != (int64_t)p->H * p->dh) return HCSA_ERR_SHAPE;   // rows are written contiguously
    if (!aligned(parts) || !aligned(out)) return HCSA_ERR_ALIGN;
    const int64_t nacc = (int64_t)p->B * p->H * p->dh, blk = nacc + 2 * (int64_t)p->B * p->H;
    return launch_merge_parts(parts, parts + nacc, blk, (int64_t)p->H * p->dh, blk / 2, p->H, n_parts, p->B, p->H,
                              p->dh, out, nullptr, nullptr, (cudaStream_t)stream);
}

hcsa_status hcsa_get_device_status(void *stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return HCSA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status_word, sizeof(int)) != cudaSuccess) return HCSA_ERR_CUDA;
    if (v != 0) {
        int zero = 0;
        if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(int)) != cudaSuccess) return HCSA_ERR_CUDA;
    }
    return (hcsa_status)v;
}

int64_t hcsa_launch_count(int32_t reset) {
    int64_t v = g_launches;
    if (reset) g_launches = 0;
    return v;
}

}  // extern "C"
