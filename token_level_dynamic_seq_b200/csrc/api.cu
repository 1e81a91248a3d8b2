// C ABI entry points (declared in include/logo.h): argument validation, TMA
// descriptor set-up and kernel launches.  No allocation, no synchronisation
// except in logo_check.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "kernels.cuh"
#include "logo.h"

namespace {

using logo::AttnParams;

thread_local char g_last_error[512] = "";

// NVTX ranges around each kernel launch, for a profiler's timeline.  Off unless
// the environment sets LOGO_NVTX=1 when the library first launches something;
// NVTX itself does nothing unless a tool has injected its library.
bool nvtx_on()
{
    static const bool on = [] {
        const char* e = std::getenv("LOGO_NVTX");
        return e && e[0] == '1';
    }();
    return on;
}

struct NvtxRange {
    const bool on;
    explicit NvtxRange(const char* name) : on(nvtx_on())
    {
        if (on) nvtxRangePushA(name);
    }
    ~NvtxRange()
    {
        if (on) nvtxRangePop();
    }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

logo_status fail(logo_status s, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return s;
}

logo_status cuda_fail(cudaError_t e, const char* what)
{
    return fail(LOGO_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Workspace layout: a 256-byte header whose first word is the device status.
constexpr size_t kWsHeaderBytes = 256;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// After the header: per-sequence counts of the threshold selection, padded to 256 bytes.
size_t counts_bytes(int nseq) { return ((size_t)nseq * 4 + 255) / 256 * 256; }

// Geometry after validation.
struct Geo {
    int B, Hq, Hkv, L, d, G, nseq, max_len;
    const int32_t* cu;
};

logo_status check_shape(const logo_shape* sh, Geo& g)
{
    if (!sh) return fail(LOGO_ERR_INVALID_ARG, "shape is NULL");
    g.B = sh->B;
    g.Hq = sh->Hq;
    g.Hkv = sh->Hkv;
    g.L = sh->L;
    g.d = sh->d;
    g.cu = sh->cu_seqlens;
    if (g.d != 64 && g.d != 128) return fail(LOGO_ERR_UNSUPPORTED, "head dim d=%d (supported: 64, 128)", g.d);
    if (g.B < 1 || g.Hq < 1 || g.Hkv < 1 || g.L < 0)
        return fail(LOGO_ERR_INVALID_ARG, "B=%d Hq=%d Hkv=%d L=%d out of range", g.B, g.Hq, g.Hkv, g.L);
    if (g.Hq % g.Hkv != 0) return fail(LOGO_ERR_INVALID_ARG, "Hq=%d is not a multiple of Hkv=%d", g.Hq, g.Hkv);
    g.G = g.Hq / g.Hkv;
    if (g.cu) {
        if (g.B != 1) return fail(LOGO_ERR_INVALID_ARG, "packed varlen layout needs B == 1 (got %d)", g.B);
        if (!aligned16(g.cu) && (reinterpret_cast<uintptr_t>(g.cu) & 3u))
            return fail(LOGO_ERR_INVALID_ARG, "cu_seqlens is not 4-byte aligned");
        if (sh->nseq < 1) return fail(LOGO_ERR_INVALID_ARG, "nseq=%d must be >= 1", sh->nseq);
        if (sh->max_seqlen < 0 || sh->max_seqlen > g.L)
            return fail(LOGO_ERR_INVALID_ARG, "max_seqlen=%d outside [0, L=%d]", sh->max_seqlen, g.L);
        g.nseq = sh->nseq;
        g.max_len = sh->max_seqlen;
    } else {
        g.nseq = g.B;
        g.max_len = g.L;
    }
    const double rows = (double)g.B * (double)(g.Hq > g.Hkv ? g.Hq : g.Hkv) * (double)g.L;
    if (rows >= 2147483647.0) return fail(LOGO_ERR_UNSUPPORTED, "B*H*L=%.0f rows exceeds 2^31-1", rows);
    return LOGO_OK;
}

logo_status check_ptr(const void* p, const char* name)
{
    if (!p) return fail(LOGO_ERR_INVALID_ARG, "%s is NULL", name);
    if (!aligned16(p)) return fail(LOGO_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return LOGO_OK;
}

logo_status check_ws(void* ws, size_t ws_bytes)
{
    if (!ws || ws_bytes < kWsHeaderBytes || !aligned16(ws))
        return fail(LOGO_ERR_WORKSPACE, "workspace %p of %zu bytes (need >= %zu, 16-byte aligned)", ws, ws_bytes,
                    kWsHeaderBytes);
    return LOGO_OK;
}

logo_status check_ratio(double ratio)
{
    if (!(ratio >= 0.0 && ratio <= 1.0)) return fail(LOGO_ERR_INVALID_ARG, "ratio=%g outside [0, 1]", ratio);
    return LOGO_OK;
}

logo_status resolve_scale(float scale, int d, float& scale_log2)
{
    if (std::isnan(scale) || std::isinf(scale)) return fail(LOGO_ERR_INVALID_ARG, "scale is not finite");
    const double s = scale > 0.f ? (double)scale : 1.0 / std::sqrt((double)d);
    scale_log2 = (float)(s * 1.4426950408889634);  // log2(e)
    return LOGO_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn(logo_status& st)
{
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    static cudaError_t err = cudaSuccess;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        err = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q);
        if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    st = fn ? LOGO_OK
            : fail(LOGO_ERR_CUDA, "cuTensorMapEncodeTiled unavailable: %s", cudaGetErrorString(err));
    return fn;
}

// 3-D bf16 view [slabs][rows][d] with a box of 64 x box_rows x 1 and the 128B swizzle.
logo_status make_map_box(CUtensorMap* map, const void* base, int d, int rows, int slabs, int box_rows)
{
    logo_status st;
    EncodeTiledFn fn = encode_fn(st);
    if (!fn) return st;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)(rows > 0 ? rows : 1), (cuuint64_t)slabs};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * 2 * (cuuint64_t)(rows > 0 ? rows : 1)};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(LOGO_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return LOGO_OK;
}

logo_status make_map(CUtensorMap* map, const void* base, int d, int rows, int slabs)
{
    return make_map_box(map, base, d, rows, slabs, 128);
}

void base_params(AttnParams& p, const Geo& g, const void* q, const void* k, const void* v, void* out,
                 float scale_log2, void* ws)
{
    memset(&p, 0, sizeof p);
    p.q = static_cast<const uint16_t*>(q);
    p.out = static_cast<uint16_t*>(out);
    p.cu_seqlens = g.cu;
    p.status = static_cast<uint32_t*>(ws);
    p.Hq = g.Hq;
    p.Hkv = g.Hkv;
    p.G = g.G;
    p.L = g.L;
    p.nseq = g.nseq;
    p.pair_heads = (g.G % 2 == 0) ? 1 : 0;
    p.scale_log2 = scale_log2;
    p.timeout_ns = 1000000000ull;  // 1 s per wait: far above any legitimate stall
    (void)k;
    (void)v;
}

// Statistics the training forward saves for the backward pass (all optional).
struct SavedStats {
    float* lse = nullptr;      // [B*Hq][L]
    float* lse_sel = nullptr;  // [Hq][sel_stride]
    uint16_t* glob = nullptr;  // [Hq][sel_stride][d]
    uint16_t* loc_sel = nullptr;  // [Hq][sel_stride][d]
    int sel_stride = 0;
};

logo_status launch_local(const Geo& g, const void* q, const void* k, const void* v, int window, float scale_log2,
                         void* out, void* ws, cudaStream_t stream, const SavedStats* saved = nullptr)
{
    if (g.L == 0 || g.max_len == 0) return LOGO_OK;
    AttnParams p;
    base_params(p, g, q, k, v, out, scale_log2, ws);
    if (saved) p.lse = saved->lse;
    p.window = window < g.max_len ? window : (g.max_len > 0 ? g.max_len : 1);
    logo_status st;
    if ((st = make_map(&p.tm_q, q, g.d, g.L, g.B * g.Hq)) != LOGO_OK) return st;
    if ((st = make_map(&p.tm_k, k, g.d, g.L, g.B * g.Hkv)) != LOGO_OK) return st;
    if ((st = make_map(&p.tm_v, v, g.d, g.L, g.B * g.Hkv)) != LOGO_OK) return st;
    NvtxRange range("logo local attention");
    cudaError_t e = logo::launch_attn(logo::kModeLocal, g.d, p, g.max_len, stream);
    if (e != cudaSuccess) return cuda_fail(e, "local attention launch");
    return LOGO_OK;
}

logo_status launch_global(const Geo& g, const void* q, const void* k, const void* v, const float* gate,
                          const int32_t* sel_idx, const int32_t* cu_sel, int max_selected, float scale_log2,
                          int merge, void* out, void* ws, cudaStream_t stream, const SavedStats* saved = nullptr)
{
    if (g.L == 0 || g.max_len == 0 || max_selected == 0) return LOGO_OK;
    AttnParams p;
    base_params(p, g, q, k, v, out, scale_log2, ws);
    if (saved) {
        p.lse = saved->lse_sel;
        p.glob = saved->glob;
        p.loc_sel = saved->loc_sel;
        p.sel_stride = saved->sel_stride;
    }
    p.gate = gate;
    p.sel_idx = sel_idx;
    p.cu_sel = cu_sel;
    p.max_selected = max_selected;
    p.merge = merge ? 1 : 0;
    p.window = g.max_len;
    logo_status st;
    if ((st = make_map(&p.tm_k, k, g.d, g.L, g.B * g.Hkv)) != LOGO_OK) return st;
    if ((st = make_map(&p.tm_v, v, g.d, g.L, g.B * g.Hkv)) != LOGO_OK) return st;
    NvtxRange range("logo selected-query global attention");
    cudaError_t e = logo::launch_attn(logo::kModeGlobal, g.d, p, g.max_len, stream);
    if (e != cudaSuccess) return cuda_fail(e, "global attention launch");
    return LOGO_OK;
}

}  // namespace

void logo::set_last_error(const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
}

namespace {

// Backward workspace: header | D of local rows | D of selected rows | row -> list slot |
// Q of selected rows | sigmoid(g) dout of selected rows | fp32 dQ of selected rows.
struct BwdWs {
    size_t dl, ds_sel, slot, q_sel, do_sel, dq_sel, total;
};

size_t round256(size_t n) { return (n + 255) / 256 * 256; }

BwdWs bwd_layout(const Geo& g, int cap)
{
    BwdWs w;
    size_t off = kWsHeaderBytes;
    const size_t rows = (size_t)g.B * g.Hq * g.L, sel = (size_t)g.Hq * (size_t)cap;
    w.dl = off;
    off += round256(rows * 4);
    w.ds_sel = off;
    off += round256(sel * 4);
    w.slot = off;
    off += round256((size_t)g.B * g.L * 4);
    w.q_sel = off;
    off += round256(sel * g.d * 2);
    w.do_sel = off;
    off += round256(sel * g.d * 2);
    w.dq_sel = off;
    off += round256(sel * g.d * 4);
    w.total = off;
    return w;
}

// ---------------------------------------------------------------- host-buffer forward
//
// Layout of the device arena of logo_forward_host (every part 256-byte aligned):
//   workspace (header + per-sequence counts) | gate | cu_seqlens (packed only) |
//   selection lists | cu_sel | kHostSlots x (Q, K, V, O of one kv-head group).
constexpr int kHostSlots = 3;

struct HostArena {
    size_t ws, gate, cu, sel, cu_sel, slot0, slot_bytes, q_bytes, kv_bytes, total, ws_bytes;
    int sel_cap;
};

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

HostArena host_arena(const Geo& g, double ratio)
{
    HostArena a;
    const int max_sel = (int)logo::budget_count(ratio, g.max_len);
    a.sel_cap = g.nseq * max_sel;
    a.ws_bytes = kWsHeaderBytes + counts_bytes(g.nseq);
    a.ws = 0;
    a.gate = up256(a.ws_bytes);
    a.cu = a.gate + up256((size_t)g.B * g.L * sizeof(float));
    a.sel = a.cu + (g.cu ? up256((size_t)(g.nseq + 1) * 4) : 0);
    a.cu_sel = a.sel + up256((size_t)(a.sel_cap > 0 ? a.sel_cap : 1) * 4);
    a.slot0 = a.cu_sel + up256((size_t)(g.nseq + 1) * 4);
    a.q_bytes = (size_t)g.B * g.G * g.L * g.d * 2;
    a.kv_bytes = (size_t)g.B * g.L * g.d * 2;
    a.slot_bytes = up256(a.q_bytes) * 2 + up256(a.kv_bytes) * 2;  // Q, O, K, V
    const int slots = g.Hkv < kHostSlots ? g.Hkv : kHostSlots;
    a.total = a.slot0 + (size_t)slots * a.slot_bytes;
    return a;
}

// Streams and events of the copy pipeline, one set per device, created on first use.
struct HostPipe {
    bool ready = false;
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t start, inputs, sel_done, h2d, comp, done, d2h[kHostSlots];
};
std::mutex g_host_mu;
HostPipe g_host_pipes[64];

cudaError_t host_pipe(int dev, HostPipe*& hp)
{
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    hp = &g_host_pipes[dev];
    if (hp->ready) return cudaSuccess;
    cudaError_t e;
    if ((e = cudaStreamCreateWithFlags(&hp->in, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithFlags(&hp->out, cudaStreamNonBlocking)) != cudaSuccess) return e;
    cudaEvent_t* evs[] = {&hp->start, &hp->inputs, &hp->sel_done, &hp->h2d, &hp->comp, &hp->done};
    for (cudaEvent_t* ev : evs)
        if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return e;
    for (int i = 0; i < kHostSlots; ++i)
        if ((e = cudaEventCreateWithFlags(&hp->d2h[i], cudaEventDisableTiming)) != cudaSuccess) return e;
    hp->ready = true;
    return cudaSuccess;
}

// `rows` copies of `row_bytes` each, source and destination rows `src_pitch` /
// `dst_pitch` bytes apart (one cudaMemcpyAsync per row).
cudaError_t copy_rows(void* dst, size_t dst_pitch, const void* src, size_t src_pitch, size_t row_bytes, int rows,
                      cudaMemcpyKind kind, cudaStream_t s)
{
    for (int r = 0; r < rows; ++r) {
        cudaError_t e = cudaMemcpyAsync(static_cast<uint8_t*>(dst) + r * dst_pitch,
                                        static_cast<const uint8_t*>(src) + r * src_pitch, row_bytes, kind, s);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

extern "C" {

int64_t logo_num_selected(double ratio, int64_t len) { return logo::budget_count(ratio, len); }

size_t logo_workspace_size(const logo_shape* shape, double ratio)
{
    Geo g;
    if (check_shape(shape, g) != LOGO_OK || check_ratio(ratio) != LOGO_OK) return 0;
    return kWsHeaderBytes + counts_bytes(g.nseq);
}

logo_status logo_workspace_init(void* ws, size_t ws_bytes, logo_stream_t stream)
{
    logo_status st = check_ws(ws, ws_bytes);
    if (st != LOGO_OK) return st;
    cudaError_t e = cudaMemsetAsync(ws, 0, kWsHeaderBytes, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? LOGO_OK : cuda_fail(e, "workspace init");
}

logo_status logo_select(const float* gate, const logo_shape* shape, double ratio, int32_t* sel_idx, int32_t* cu_sel,
                        void* ws, size_t ws_bytes, logo_stream_t stream)
{
    Geo g;
    logo_status st;
    if ((st = check_shape(shape, g)) != LOGO_OK) return st;
    if ((st = check_ratio(ratio)) != LOGO_OK) return st;
    if ((st = check_ws(ws, ws_bytes)) != LOGO_OK) return st;
    if ((st = check_ptr(cu_sel, "cu_sel")) != LOGO_OK) return st;
    if (g.L > 0 && (st = check_ptr(gate, "gate")) != LOGO_OK) return st;
    if (g.L > 0 && logo::budget_count(ratio, g.max_len) > 0 && (st = check_ptr(sel_idx, "sel_idx")) != LOGO_OK)
        return st;
    cudaError_t e;
    if (g.L == 0 && !g.cu) {
        e = cudaMemsetAsync(cu_sel, 0, sizeof(int32_t) * (size_t)(g.nseq + 1), static_cast<cudaStream_t>(stream));
    } else {
        NvtxRange range("logo select");
        e = logo::launch_select(gate, g.cu, g.nseq, g.L, g.max_len, ratio, sel_idx, cu_sel,
                                static_cast<cudaStream_t>(stream));
    }
    return e == cudaSuccess ? LOGO_OK : cuda_fail(e, "select launch");
}

logo_status logo_local_attn(const logo_bf16* q, const logo_bf16* k, const logo_bf16* v, const logo_shape* shape,
                            int window, float scale, logo_bf16* out, void* ws, size_t ws_bytes, logo_stream_t stream)
{
    Geo g;
    logo_status st;
    float sl2;
    if ((st = check_shape(shape, g)) != LOGO_OK) return st;
    if (window < 1) return fail(LOGO_ERR_INVALID_ARG, "window=%d must be >= 1", window);
    if ((st = resolve_scale(scale, g.d, sl2)) != LOGO_OK) return st;
    if ((st = check_ws(ws, ws_bytes)) != LOGO_OK) return st;
    if (g.L > 0) {
        if ((st = check_ptr(q, "q")) != LOGO_OK || (st = check_ptr(k, "k")) != LOGO_OK ||
            (st = check_ptr(v, "v")) != LOGO_OK || (st = check_ptr(out, "out")) != LOGO_OK)
            return st;
    }
    return launch_local(g, q, k, v, window, sl2, out, ws, static_cast<cudaStream_t>(stream));
}

logo_status logo_global_attn_sparse(const logo_bf16* q, const logo_bf16* k, const logo_bf16* v, const float* gate,
                                    const int32_t* sel_idx, const int32_t* cu_sel, const logo_shape* shape,
                                    int max_selected, float scale, int merge, logo_bf16* out, void* ws,
                                    size_t ws_bytes, logo_stream_t stream)
{
    Geo g;
    logo_status st;
    float sl2;
    if ((st = check_shape(shape, g)) != LOGO_OK) return st;
    if ((st = resolve_scale(scale, g.d, sl2)) != LOGO_OK) return st;
    if ((st = check_ws(ws, ws_bytes)) != LOGO_OK) return st;
    if (max_selected < 0 || max_selected > g.max_len)
        return fail(LOGO_ERR_INVALID_ARG, "max_selected=%d outside [0, %d]", max_selected, g.max_len);
    if (g.L > 0 && max_selected > 0) {
        if ((st = check_ptr(q, "q")) != LOGO_OK || (st = check_ptr(k, "k")) != LOGO_OK ||
            (st = check_ptr(v, "v")) != LOGO_OK || (st = check_ptr(out, "out")) != LOGO_OK ||
            (st = check_ptr(sel_idx, "sel_idx")) != LOGO_OK || (st = check_ptr(cu_sel, "cu_sel")) != LOGO_OK)
            return st;
        if (merge && (st = check_ptr(gate, "gate")) != LOGO_OK) return st;
    }
    return launch_global(g, q, k, v, gate, sel_idx, cu_sel, max_selected, sl2, merge, out, ws,
                         static_cast<cudaStream_t>(stream));
}

logo_status logo_forward(const logo_bf16* q, const logo_bf16* k, const logo_bf16* v, const float* gate,
                         const logo_shape* shape, int window, double ratio, float scale, logo_bf16* out,
                         int32_t* sel_idx, int32_t* cu_sel, void* ws, size_t ws_bytes, logo_stream_t stream)
{
    Geo g;
    logo_status st;
    float sl2;
    if ((st = check_shape(shape, g)) != LOGO_OK) return st;
    if ((st = check_ratio(ratio)) != LOGO_OK) return st;
    if (window < 1) return fail(LOGO_ERR_INVALID_ARG, "window=%d must be >= 1", window);
    if ((st = resolve_scale(scale, g.d, sl2)) != LOGO_OK) return st;
    if ((st = check_ws(ws, ws_bytes)) != LOGO_OK) return st;
    if ((st = check_ptr(cu_sel, "cu_sel")) != LOGO_OK) return st;
    const int max_sel = (int)logo::budget_count(ratio, g.max_len);
    if (g.L > 0) {
        if ((st = check_ptr(q, "q")) != LOGO_OK || (st = check_ptr(k, "k")) != LOGO_OK ||
            (st = check_ptr(v, "v")) != LOGO_OK || (st = check_ptr(out, "out")) != LOGO_OK ||
            (st = check_ptr(gate, "gate")) != LOGO_OK)
            return st;
        if (max_sel > 0 && (st = check_ptr(sel_idx, "sel_idx")) != LOGO_OK) return st;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = logo_select(gate, shape, ratio, sel_idx, cu_sel, ws, ws_bytes, stream)) != LOGO_OK) return st;
    if ((st = launch_local(g, q, k, v, window, sl2, out, ws, s)) != LOGO_OK) return st;
    return launch_global(g, q, k, v, gate, sel_idx, cu_sel, max_sel, sl2, 1, out, ws, s);
}

logo_status logo_forward_train(const logo_bf16* q, const logo_bf16* k, const logo_bf16* v, const float* gate,
                               const logo_shape* shape, int window, double ratio, float scale, logo_bf16* out,
                               int32_t* sel_idx, int32_t* cu_sel, int sel_capacity, float* lse, float* lse_sel,
                               logo_bf16* glob, logo_bf16* loc_sel, void* ws, size_t ws_bytes, logo_stream_t stream)
{
    Geo g;
    logo_status st;
    float sl2;
    if ((st = check_shape(shape, g)) != LOGO_OK) return st;
    if ((st = check_ratio(ratio)) != LOGO_OK) return st;
    if (window < 1) return fail(LOGO_ERR_INVALID_ARG, "window=%d must be >= 1", window);
    if ((st = resolve_scale(scale, g.d, sl2)) != LOGO_OK) return st;
    if ((st = check_ws(ws, ws_bytes)) != LOGO_OK) return st;
    if ((st = check_ptr(cu_sel, "cu_sel")) != LOGO_OK) return st;
    const int max_sel = (int)logo::budget_count(ratio, g.max_len);
    if (sel_capacity < 0) return fail(LOGO_ERR_INVALID_ARG, "sel_capacity=%d must be >= 0", sel_capacity);
    if (max_sel > 0 && sel_capacity < max_sel)
        return fail(LOGO_ERR_INVALID_ARG, "sel_capacity=%d is below one sequence's count %d", sel_capacity, max_sel);
    if (g.L > 0) {
        if ((st = check_ptr(q, "q")) != LOGO_OK || (st = check_ptr(k, "k")) != LOGO_OK ||
            (st = check_ptr(v, "v")) != LOGO_OK || (st = check_ptr(out, "out")) != LOGO_OK ||
            (st = check_ptr(gate, "gate")) != LOGO_OK || (st = check_ptr(lse, "lse")) != LOGO_OK)
            return st;
        if (max_sel > 0 && ((st = check_ptr(sel_idx, "sel_idx")) != LOGO_OK ||
                            (st = check_ptr(lse_sel, "lse_sel")) != LOGO_OK || (st = check_ptr(glob, "glob")) != LOGO_OK ||
                            (st = check_ptr(loc_sel, "loc_sel")) != LOGO_OK))
            return st;
    }
    SavedStats saved;
    saved.lse = lse;
    saved.lse_sel = lse_sel;
    saved.glob = reinterpret_cast<uint16_t*>(glob);
    saved.loc_sel = reinterpret_cast<uint16_t*>(loc_sel);
    saved.sel_stride = sel_capacity;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = logo_select(gate, shape, ratio, sel_idx, cu_sel, ws, ws_bytes, stream)) != LOGO_OK) return st;
    if ((st = launch_local(g, q, k, v, window, sl2, out, ws, s, &saved)) != LOGO_OK) return st;
    return launch_global(g, q, k, v, gate, sel_idx, cu_sel, max_sel, sl2, 1, out, ws, s, &saved);
}

size_t logo_backward_workspace_size(const logo_shape* shape, int sel_capacity)
{
    Geo g;
    if (check_shape(shape, g) != LOGO_OK || sel_capacity < 0) return 0;
    return bwd_layout(g, sel_capacity).total;
}

logo_status logo_backward(const logo_bf16* q, const logo_bf16* k, const logo_bf16* v, const float* gate,
                          const logo_bf16* out, const logo_bf16* dout, const int32_t* sel_idx, const int32_t* cu_sel,
                          int sel_capacity, int max_selected, const float* lse, const float* lse_sel,
                          const logo_bf16* glob, const logo_bf16* loc_sel, const logo_shape* shape, int window,
                          float scale, logo_bf16* dq,
                          logo_bf16* dk, logo_bf16* dv, float* dgate, void* ws, size_t ws_bytes,
                          logo_stream_t stream)
{
    Geo g;
    logo_status st;
    float sl2;
    if ((st = check_shape(shape, g)) != LOGO_OK) return st;
    if (window < 1) return fail(LOGO_ERR_INVALID_ARG, "window=%d must be >= 1", window);
    if ((st = resolve_scale(scale, g.d, sl2)) != LOGO_OK) return st;
    if (sel_capacity < 0) return fail(LOGO_ERR_INVALID_ARG, "sel_capacity=%d must be >= 0", sel_capacity);
    if (max_selected < 0 || max_selected > g.max_len || max_selected > sel_capacity)
        return fail(LOGO_ERR_INVALID_ARG, "max_selected=%d outside [0, min(%d, sel_capacity=%d)]", max_selected,
                    g.max_len, sel_capacity);
    if ((st = check_ws(ws, ws_bytes)) != LOGO_OK) return st;
    const BwdWs lay = bwd_layout(g, sel_capacity);
    if (ws_bytes < lay.total)
        return fail(LOGO_ERR_WORKSPACE, "backward workspace of %zu bytes, need %zu", ws_bytes, lay.total);
    if (g.L == 0 || g.max_len == 0) return LOGO_OK;
    if ((st = check_ptr(q, "q")) != LOGO_OK || (st = check_ptr(k, "k")) != LOGO_OK ||
        (st = check_ptr(v, "v")) != LOGO_OK || (st = check_ptr(gate, "gate")) != LOGO_OK ||
        (st = check_ptr(out, "out")) != LOGO_OK || (st = check_ptr(dout, "dout")) != LOGO_OK ||
        (st = check_ptr(lse, "lse")) != LOGO_OK || (st = check_ptr(cu_sel, "cu_sel")) != LOGO_OK ||
        (st = check_ptr(dq, "dq")) != LOGO_OK || (st = check_ptr(dk, "dk")) != LOGO_OK ||
        (st = check_ptr(dv, "dv")) != LOGO_OK || (st = check_ptr(dgate, "dgate")) != LOGO_OK)
        return st;
    const bool any_sel = max_selected > 0;
    if (any_sel && ((st = check_ptr(sel_idx, "sel_idx")) != LOGO_OK || (st = check_ptr(lse_sel, "lse_sel")) != LOGO_OK ||
                    (st = check_ptr(glob, "glob")) != LOGO_OK || (st = check_ptr(loc_sel, "loc_sel")) != LOGO_OK))
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* wb = static_cast<uint8_t*>(ws);
    float* dl = reinterpret_cast<float*>(wb + lay.dl);
    float* ds_sel = reinterpret_cast<float*>(wb + lay.ds_sel);
    int32_t* slot = reinterpret_cast<int32_t*>(wb + lay.slot);
    uint16_t* q_sel = reinterpret_cast<uint16_t*>(wb + lay.q_sel);
    uint16_t* do_sel = reinterpret_cast<uint16_t*>(wb + lay.do_sel);
    float* dq_sel = reinterpret_cast<float*>(wb + lay.dq_sel);

    logo::PrepParams pp;
    memset(&pp, 0, sizeof pp);
    pp.q = static_cast<const uint16_t*>(q);
    pp.out = static_cast<const uint16_t*>(out);
    pp.dout = static_cast<const uint16_t*>(dout);
    pp.glob = static_cast<const uint16_t*>(glob);
    pp.loc_sel = static_cast<const uint16_t*>(loc_sel);
    pp.gate = gate;
    pp.cu_seqlens = g.cu;
    pp.sel_idx = sel_idx;
    pp.cu_sel = any_sel ? cu_sel : nullptr;
    pp.dl = dl;
    pp.ds_sel = ds_sel;
    pp.dgate = dgate;
    pp.slot = slot;
    pp.q_sel = q_sel;
    pp.do_sel = do_sel;
    pp.status = static_cast<uint32_t*>(ws);
    pp.B = g.B;
    pp.Hq = g.Hq;
    pp.L = g.L;
    pp.nseq = g.nseq;
    pp.sel_stride = any_sel ? sel_capacity : 0;
    NvtxRange range("logo backward");
    cudaError_t e = logo::launch_bwd_prep(pp, g.d, s);
    if (e != cudaSuccess) return cuda_fail(e, "backward prep launch");

    logo::BwdParams p;
    memset(&p, 0, sizeof p);
    if ((st = make_map(&p.tm_q, q, g.d, g.L, g.B * g.Hq)) != LOGO_OK) return st;
    if ((st = make_map(&p.tm_do, dout, g.d, g.L, g.B * g.Hq)) != LOGO_OK) return st;
    if ((st = make_map(&p.tm_k, k, g.d, g.L, g.B * g.Hkv)) != LOGO_OK) return st;
    if ((st = make_map(&p.tm_v, v, g.d, g.L, g.B * g.Hkv)) != LOGO_OK) return st;
    if (any_sel) {
        if ((st = make_map(&p.tm_qs, q_sel, g.d, sel_capacity, g.Hq)) != LOGO_OK) return st;
        if ((st = make_map(&p.tm_dos, do_sel, g.d, sel_capacity, g.Hq)) != LOGO_OK) return st;
    }
    p.lse = lse;
    p.dl = dl;
    p.lse_s = lse_sel;
    p.ds_sel = ds_sel;
    p.cu_seqlens = g.cu;
    p.sel_idx = sel_idx;
    p.cu_sel = cu_sel;
    p.slot = slot;
    p.dq_sel = any_sel ? dq_sel : nullptr;
    p.dq = reinterpret_cast<uint16_t*>(dq);
    p.dk = reinterpret_cast<uint16_t*>(dk);
    p.dv = reinterpret_cast<uint16_t*>(dv);
    p.status = static_cast<uint32_t*>(ws);
    p.Hq = g.Hq;
    p.Hkv = g.Hkv;
    p.G = g.G;
    p.L = g.L;
    p.nseq = g.nseq;
    p.window = window < g.max_len ? window : g.max_len;
    p.max_selected = max_selected;
    p.sel_stride = sel_capacity;
    p.scale_log2 = sl2;
    p.scale = scale > 0.f ? scale : (float)(1.0 / std::sqrt((double)g.d));
    p.timeout_ns = 1000000000ull;
    if (any_sel && (e = logo::launch_bwd_dq(logo::kModeGlobal, g.d, p, g.max_len, s)) != cudaSuccess)
        return cuda_fail(e, "backward dQ (selected rows) launch");
    if ((e = logo::launch_bwd_dq(logo::kModeLocal, g.d, p, g.max_len, s)) != cudaSuccess)
        return cuda_fail(e, "backward dQ launch");
    if ((e = logo::launch_bwd_dkdv(g.d, p, g.max_len, s)) != cudaSuccess)
        return cuda_fail(e, "backward dK/dV launch");
    return LOGO_OK;
}

logo_status logo_select_threshold(const float* gate, const logo_shape* shape, const float* tau, int max_selected,
                                  int32_t* sel_idx, int32_t* cu_sel, void* ws, size_t ws_bytes, logo_stream_t stream)
{
    Geo g;
    logo_status st;
    if ((st = check_shape(shape, g)) != LOGO_OK) return st;
    if ((st = check_ws(ws, ws_bytes)) != LOGO_OK) return st;
    if (ws_bytes < kWsHeaderBytes + counts_bytes(g.nseq))
        return fail(LOGO_ERR_WORKSPACE, "workspace of %zu bytes, the threshold selection needs %zu", ws_bytes,
                    kWsHeaderBytes + counts_bytes(g.nseq));
    if (max_selected < 0 || max_selected > g.max_len)
        return fail(LOGO_ERR_INVALID_ARG, "max_selected=%d outside [0, %d]", max_selected, g.max_len);
    if ((st = check_ptr(cu_sel, "cu_sel")) != LOGO_OK) return st;
    if ((st = check_ptr(tau, "tau")) != LOGO_OK) return st;
    if (g.L > 0 && (st = check_ptr(gate, "gate")) != LOGO_OK) return st;
    if (max_selected > 0 && (st = check_ptr(sel_idx, "sel_idx")) != LOGO_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* counts = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + kWsHeaderBytes);
    NvtxRange range("logo threshold select");
    cudaError_t e = logo::launch_threshold_select(gate, g.cu, g.nseq, g.L, g.max_len, tau, max_selected, counts,
                                                  sel_idx, cu_sel, static_cast<uint32_t*>(ws), s);
    return e == cudaSuccess ? LOGO_OK : cuda_fail(e, "threshold select launch");
}

logo_status logo_threshold_update(const float* gate, const logo_shape* shape, double ratio, float beta, float* tau,
                                  float* target, void* ws, size_t ws_bytes, logo_stream_t stream)
{
    Geo g;
    logo_status st;
    if ((st = check_shape(shape, g)) != LOGO_OK) return st;
    if ((st = check_ratio(ratio)) != LOGO_OK) return st;
    if ((st = check_ws(ws, ws_bytes)) != LOGO_OK) return st;
    if (std::isnan(beta) || beta < 0.f || beta > 1.f) return fail(LOGO_ERR_INVALID_ARG, "beta=%g outside [0, 1]", beta);
    if ((st = check_ptr(tau, "tau")) != LOGO_OK) return st;
    if (target && (reinterpret_cast<uintptr_t>(target) & 3u))
        return fail(LOGO_ERR_INVALID_ARG, "target is not 4-byte aligned");
    if (g.L > 0 && (st = check_ptr(gate, "gate")) != LOGO_OK) return st;
    const long long n_fixed = (long long)g.B * g.L;
    NvtxRange range("logo threshold update");
    const long long n_all = g.cu ? (long long)g.L : n_fixed;  // packed: L is the total token count
    cudaError_t e = logo::launch_threshold_update(gate, g.cu, g.nseq, n_all, n_fixed, ratio, beta, tau, target,
                                                  static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? LOGO_OK : cuda_fail(e, "threshold update launch");
}

size_t logo_decode_workspace_size(const logo_shape* shape)
{
    Geo g;
    if (check_shape(shape, g) != LOGO_OK || g.cu) return 0;
    return kWsHeaderBytes + logo::decode_partials_bytes(g.B, g.Hkv, g.G, g.L, g.d);
}

logo_status logo_decode(const logo_bf16* q, const logo_bf16* k_cache, const logo_bf16* v_cache,
                        const int32_t* cache_len, const float* gate, const float* tau, const logo_shape* shape,
                        int window, float scale, logo_bf16* out, int32_t* selected, void* ws, size_t ws_bytes,
                        logo_stream_t stream)
{
    Geo g;
    logo_status st;
    float sl2;
    if ((st = check_shape(shape, g)) != LOGO_OK) return st;
    if (g.cu) return fail(LOGO_ERR_INVALID_ARG, "decode takes one cache per sequence (cu_seqlens must be NULL)");
    if (g.G != 1 && g.G != 2 && g.G != 4 && g.G != 8)
        return fail(LOGO_ERR_UNSUPPORTED, "decode supports Hq/Hkv in {1, 2, 4, 8} (got %d)", g.G);
    if (window < 1) return fail(LOGO_ERR_INVALID_ARG, "window=%d must be >= 1", window);
    if ((st = resolve_scale(scale, g.d, sl2)) != LOGO_OK) return st;
    if ((st = check_ws(ws, ws_bytes)) != LOGO_OK) return st;
    const size_t need = kWsHeaderBytes + logo::decode_partials_bytes(g.B, g.Hkv, g.G, g.L, g.d);
    if (ws_bytes < need) return fail(LOGO_ERR_WORKSPACE, "workspace of %zu bytes, decode needs %zu", ws_bytes, need);
    if ((st = check_ptr(q, "q")) != LOGO_OK || (st = check_ptr(out, "out")) != LOGO_OK ||
        (st = check_ptr(cache_len, "cache_len")) != LOGO_OK || (st = check_ptr(gate, "gate")) != LOGO_OK ||
        (st = check_ptr(tau, "tau")) != LOGO_OK)
        return st;
    if (g.L > 0 && ((st = check_ptr(k_cache, "k_cache")) != LOGO_OK || (st = check_ptr(v_cache, "v_cache")) != LOGO_OK))
        return st;
    if (selected && (reinterpret_cast<uintptr_t>(selected) & 3u))
        return fail(LOGO_ERR_INVALID_ARG, "selected is not 4-byte aligned");
    logo::DecodeParams p;
    memset(&p, 0, sizeof p);
    p.q = reinterpret_cast<const uint16_t*>(q);
    p.k = reinterpret_cast<const uint16_t*>(k_cache);
    p.v = reinterpret_cast<const uint16_t*>(v_cache);
    p.cache_len = cache_len;
    p.gate = gate;
    p.tau = tau;
    p.out = reinterpret_cast<uint16_t*>(out);
    p.selected = selected;
    p.part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kWsHeaderBytes);
    p.status = static_cast<uint32_t*>(ws);
    p.B = g.B;
    p.Hq = g.Hq;
    p.Hkv = g.Hkv;
    p.G = g.G;
    p.Lmax = g.L;
    p.d = g.d;
    p.W = window < g.L ? window : (g.L > 0 ? g.L : 1);
    p.chunk = logo::kDecChunk;
    p.nchunks = g.L > 0 ? (g.L + logo::kDecChunk - 1) / logo::kDecChunk : 1;
    p.scale_log2 = sl2;
    p.timeout_ns = 1000000000ull;  // 1 s per wait: far above any legitimate stall
    if (g.L > 0) {
        if ((st = make_map_box(&p.tm_k, k_cache, g.d, g.L, g.B * g.Hkv, logo::kDecBlock)) != LOGO_OK ||
            (st = make_map_box(&p.tm_v, v_cache, g.d, g.L, g.B * g.Hkv, logo::kDecBlock)) != LOGO_OK)
            return st;
    }
    NvtxRange range("logo decode");
    cudaError_t e = logo::launch_decode(p, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? LOGO_OK : cuda_fail(e, "decode launch");
}

logo_status logo_check(const void* ws, logo_stream_t stream)
{
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "pending launch error");
    if (!ws) return fail(LOGO_ERR_WORKSPACE, "workspace is NULL");
    uint32_t status = 0;
    e = cudaMemcpy(&status, ws, sizeof status, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "status read");
    if (status & logo::kStatusTimeout)
        return fail(LOGO_ERR_DEVICE_TIMEOUT, "a kernel's bounded wait ran out (status 0x%x)", status);
    if (status & logo::kStatusBadArgument)
        return fail(LOGO_ERR_INVALID_ARG, "a kernel met an argument it cannot handle (status 0x%x)", status);
    if (status & logo::kStatusBounds)
        return fail(LOGO_ERR_BOUNDS, "a debug bounds check failed and skipped an access (status 0x%x)", status);
    if (status & logo::kStatusCapacity)
        return fail(LOGO_ERR_CAPACITY, "more tokens passed the threshold than max_selected (status 0x%x)", status);
    return LOGO_OK;
}

logo_status logo_selftest_timeout(void* ws, size_t ws_bytes, unsigned limit_us, logo_stream_t stream)
{
    logo_status st = check_ws(ws, ws_bytes);
    if (st != LOGO_OK) return st;
    if (limit_us == 0 || limit_us > 10000000u)
        return fail(LOGO_ERR_INVALID_ARG, "limit_us=%u outside [1, 10^7]", limit_us);
    cudaError_t e = logo::launch_timeout_probe(static_cast<uint32_t*>(ws), 1000ull * limit_us,
                                               static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? LOGO_OK : cuda_fail(e, "timeout probe launch");
}

size_t logo_forward_host_buffer_size(const logo_shape* shape, double ratio)
{
    Geo g;
    if (check_shape(shape, g) != LOGO_OK || check_ratio(ratio) != LOGO_OK) return 0;
    return host_arena(g, ratio).total;
}

logo_status logo_forward_host(const logo_bf16* q, const logo_bf16* k, const logo_bf16* v, const float* gate,
                              const logo_shape* shape, int window, double ratio, float scale, logo_bf16* out,
                              int32_t* sel_idx, int32_t* cu_sel, void* dev_buf, size_t dev_buf_bytes,
                              logo_stream_t stream)
{
    Geo g;
    logo_status st;
    float sl2;
    if ((st = check_shape(shape, g)) != LOGO_OK) return st;
    if ((st = check_ratio(ratio)) != LOGO_OK) return st;
    if (window < 1) return fail(LOGO_ERR_INVALID_ARG, "window=%d must be >= 1", window);
    if ((st = resolve_scale(scale, g.d, sl2)) != LOGO_OK) return st;
    const HostArena a = host_arena(g, ratio);
    if (!dev_buf || !aligned16(dev_buf)) return fail(LOGO_ERR_WORKSPACE, "dev_buf is NULL or not 16-byte aligned");
    if (dev_buf_bytes < a.total)
        return fail(LOGO_ERR_WORKSPACE, "dev_buf of %zu bytes, the host-buffer forward needs %zu", dev_buf_bytes, a.total);
    if (g.L > 0 && (!q || !k || !v || !out || !gate))
        return fail(LOGO_ERR_INVALID_ARG, "q, k, v, gate and out must be non-NULL host buffers");
    const int max_sel = (int)logo::budget_count(ratio, g.max_len);
    uint8_t* base = static_cast<uint8_t*>(dev_buf);
    void* ws = base + a.ws;
    float* gate_d = reinterpret_cast<float*>(base + a.gate);
    int32_t* cu_d = g.cu ? reinterpret_cast<int32_t*>(base + a.cu) : nullptr;
    int32_t* sel_d = reinterpret_cast<int32_t*>(base + a.sel);
    int32_t* cu_sel_d = reinterpret_cast<int32_t*>(base + a.cu_sel);
    cudaStream_t s0 = static_cast<cudaStream_t>(stream);

    std::lock_guard<std::mutex> lock(g_host_mu);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    HostPipe* hp = nullptr;
    if (e == cudaSuccess) e = host_pipe(dev, hp);
    if (e != cudaSuccess) return cuda_fail(e, "host pipeline setup");
#define LOGO_CK(call, what)                                   \
    do {                                                      \
        cudaError_t ce_ = (call);                             \
        if (ce_ != cudaSuccess) return cuda_fail(ce_, what);  \
    } while (0)
    // Everything the caller queued on `stream` comes first.
    LOGO_CK(cudaEventRecord(hp->start, s0), "event");
    LOGO_CK(cudaStreamWaitEvent(hp->in, hp->start, 0), "stream wait");
    LOGO_CK(cudaStreamWaitEvent(hp->out, hp->start, 0), "stream wait");
    // Gate (and packed lengths) in, selection on the compute stream.
    if (g.L > 0) LOGO_CK(cudaMemcpyAsync(gate_d, gate, (size_t)g.B * g.L * sizeof(float), cudaMemcpyHostToDevice, hp->in), "gate copy");
    if (g.cu) LOGO_CK(cudaMemcpyAsync(cu_d, g.cu, (size_t)(g.nseq + 1) * 4, cudaMemcpyHostToDevice, hp->in), "cu_seqlens copy");
    LOGO_CK(cudaEventRecord(hp->inputs, hp->in), "event");
    LOGO_CK(cudaStreamWaitEvent(s0, hp->inputs, 0), "stream wait");
    logo_shape dsh = *shape;
    dsh.cu_seqlens = cu_d;
    if ((st = logo_select(gate_d, &dsh, ratio, sel_d, cu_sel_d, ws, a.ws_bytes, stream)) != LOGO_OK) return st;
    if (sel_idx || cu_sel) {
        LOGO_CK(cudaEventRecord(hp->sel_done, s0), "event");
        LOGO_CK(cudaStreamWaitEvent(hp->out, hp->sel_done, 0), "stream wait");
        if (cu_sel) LOGO_CK(cudaMemcpyAsync(cu_sel, cu_sel_d, (size_t)(g.nseq + 1) * 4, cudaMemcpyDeviceToHost, hp->out), "cu_sel copy");
        if (sel_idx && a.sel_cap > 0)
            LOGO_CK(cudaMemcpyAsync(sel_idx, sel_d, (size_t)a.sel_cap * 4, cudaMemcpyDeviceToHost, hp->out), "sel_idx copy");
    }
    // One kv-head group at a time: its Q, K, V in, both branches, its O out, with
    // the copies of neighbouring groups overlapping the kernels.
    Geo gu = g;
    gu.Hq = g.G;
    gu.Hkv = 1;
    gu.cu = cu_d;  // the kernels read the device copy of the packed offsets
    const size_t elt = 2;
    const size_t rowq = (size_t)g.L * g.d * elt;  // one head of one sequence
    const int slots = g.Hkv < kHostSlots ? g.Hkv : kHostSlots;
    for (int hk = 0; hk < g.Hkv && g.L > 0; ++hk) {
        const int sl = hk % slots;
        uint8_t* slot = base + a.slot0 + (size_t)sl * a.slot_bytes;
        uint8_t* qs = slot;
        uint8_t* os = slot + up256(a.q_bytes);
        uint8_t* ks = os + up256(a.q_bytes);
        uint8_t* vs = ks + up256(a.kv_bytes);
        if (hk >= slots) LOGO_CK(cudaStreamWaitEvent(hp->in, hp->d2h[sl], 0), "stream wait");
        LOGO_CK(copy_rows(qs, g.G * rowq, reinterpret_cast<const uint8_t*>(q) + (size_t)hk * g.G * rowq, g.Hq * rowq,
                          g.G * rowq, g.B, cudaMemcpyHostToDevice, hp->in), "q copy");
        LOGO_CK(copy_rows(ks, rowq, reinterpret_cast<const uint8_t*>(k) + (size_t)hk * rowq, g.Hkv * rowq, rowq, g.B,
                          cudaMemcpyHostToDevice, hp->in), "k copy");
        LOGO_CK(copy_rows(vs, rowq, reinterpret_cast<const uint8_t*>(v) + (size_t)hk * rowq, g.Hkv * rowq, rowq, g.B,
                          cudaMemcpyHostToDevice, hp->in), "v copy");
        LOGO_CK(cudaEventRecord(hp->h2d, hp->in), "event");
        LOGO_CK(cudaStreamWaitEvent(s0, hp->h2d, 0), "stream wait");
        if ((st = launch_local(gu, qs, ks, vs, window, sl2, os, ws, s0)) != LOGO_OK) return st;
        if ((st = launch_global(gu, qs, ks, vs, gate_d, sel_d, cu_sel_d, max_sel, sl2, 1, os, ws, s0)) != LOGO_OK)
            return st;
        LOGO_CK(cudaEventRecord(hp->comp, s0), "event");
        LOGO_CK(cudaStreamWaitEvent(hp->out, hp->comp, 0), "stream wait");
        LOGO_CK(copy_rows(reinterpret_cast<uint8_t*>(out) + (size_t)hk * g.G * rowq, g.Hq * rowq, os, g.G * rowq,
                          g.G * rowq, g.B, cudaMemcpyDeviceToHost, hp->out), "out copy");
        LOGO_CK(cudaEventRecord(hp->d2h[sl], hp->out), "event");
    }
    // The caller's stream completes after the last copy out.
    LOGO_CK(cudaEventRecord(hp->done, hp->out), "event");
    LOGO_CK(cudaStreamWaitEvent(s0, hp->done, 0), "stream wait");
#undef LOGO_CK
    return LOGO_OK;
}

const char* logo_status_string(logo_status s)
{
    switch (s) {
        case LOGO_OK: return "LOGO_OK";
        case LOGO_ERR_INVALID_ARG: return "LOGO_ERR_INVALID_ARG";
        case LOGO_ERR_UNSUPPORTED: return "LOGO_ERR_UNSUPPORTED";
        case LOGO_ERR_WORKSPACE: return "LOGO_ERR_WORKSPACE";
        case LOGO_ERR_CUDA: return "LOGO_ERR_CUDA";
        case LOGO_ERR_DEVICE_TIMEOUT: return "LOGO_ERR_DEVICE_TIMEOUT";
        case LOGO_ERR_CAPACITY: return "LOGO_ERR_CAPACITY";
        case LOGO_ERR_BOUNDS: return "LOGO_ERR_BOUNDS";
    }
    return "LOGO_ERR_UNKNOWN";
}

const char* logo_last_error(void) { return g_last_error; }

unsigned logo_build_flags(void)
{
#ifdef LOGO_DEBUG_BOUNDS
    return LOGO_BUILD_DEBUG_BOUNDS;
#else
    return 0u;
#endif
}

}  // extern "C"
