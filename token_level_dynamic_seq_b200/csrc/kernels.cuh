// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace logo {

// Device-side status word bits (first word of the caller's workspace).
enum : uint32_t {
    kStatusTimeout = 1u,      // a bounded wait ran out
    kStatusBadArgument = 2u,  // a kernel met an argument it cannot handle
    kStatusCapacity = 4u,     // more tokens above the threshold than the output holds
    kStatusBounds = 8u,       // debug build: an index check failed and the access was skipped
};

// Budget count, identical on host and device (see logo_num_selected in
// logo.h).  The product is formed with an explicit round-to-nearest multiply
// so device code cannot contract it into a fused multiply-add.
__host__ __device__ inline int64_t budget_count(double ratio, int64_t len)
{
    if (len <= 0 || !(ratio > 0.0)) return 0;
#ifdef __CUDA_ARCH__
    const double x = __dmul_rn(ratio, (double)len);
    const double r = rint(x);
    const double diff = fabs(__dadd_rn(x, -r));
#else
    volatile double xv = ratio * (double)len;  // no contraction on the host either
    const double x = xv;
    const double r = nearbyint(x);
    const double diff = fabs(x - r);
#endif
    const double tol = 1e-9 * (x > 1.0 ? x : 1.0);
    double kk = (diff <= tol) ? r : ceil(x);
    if (kk < 0.0) kk = 0.0;
    if (kk > (double)len) kk = (double)len;
    return (int64_t)kk;
}

constexpr int kTileM = 128;   // query rows per Q tile (= TMEM lanes)
constexpr int kTileN = 128;   // keys per K/V tile
constexpr int kNumQ = 2;      // Q tiles per CTA, one softmax warpgroup each
constexpr int kThreads = 128 + 128 * kNumQ;  // producer warpgroup (TMA, MMA, 2 idle), one warpgroup per query tile
// Registers per thread after the producer warpgroup hands its share to the softmax
// warpgroups (setmaxnreg).  The launch holds kThreads * 168 (the compiler's count
// under __launch_bounds__(kThreads, 1)); the split must not exceed it, or the
// increase would wait for registers that never come free.
constexpr int kProducerRegs = 88;
constexpr int kSoftmaxRegs = 208;
static_assert(128 * kProducerRegs + 128 * kNumQ * kSoftmaxRegs <= kThreads * 168, "register split above the launch total");

enum AttnMode : int { kModeLocal = 0, kModeGlobal = 1 };

struct alignas(64) AttnParams {
    CUtensorMap tm_q;   // Q as [B*Hq][L][d] (local mode loads Q tiles by TMA)
    CUtensorMap tm_k;   // K as [B*Hkv][L][d]
    CUtensorMap tm_v;   // V as [B*Hkv][L][d]
    const uint16_t* q;  // raw Q (global mode gathers selected rows)
    uint16_t* out;
    const float* gate;
    const int32_t* cu_seqlens;  // nullptr: fixed length
    const int32_t* sel_idx;
    const int32_t* cu_sel;
    uint32_t* status;
    int Hq, Hkv, G;
    int L;          // rows per head slab (L, or T when packed)
    int nseq;
    int window;
    int pair_heads; // 1: the CTA's Q tiles are heads (h, h+1) on the same rows
    int max_selected;
    int merge;
    float scale_log2;  // softmax scale * log2(e)
    unsigned long long timeout_ns;
    // Statistics for the backward pass (training forward); nullptr: not saved.
    //   local mode:  lse [B*Hq][L]        log-sum-exp per row, log2 units of the scaled score
    //   global mode: lse [Hq][sel_stride] per selected row, glob [Hq][sel_stride][d] the global
    //                branch (bf16, before the gate), loc_sel [Hq][sel_stride][d] the local branch
    //                of the selected rows (bf16, as the local kernel wrote it), rows indexed like sel_idx
    float* lse;
    uint16_t* glob;
    uint16_t* loc_sel;
    int sel_stride;
};

cudaError_t launch_select(const float* gate, const int32_t* cu_seqlens, int nseq, int L, int max_len,
                          double ratio, int32_t* sel_idx, int32_t* cu_sel, cudaStream_t stream);

cudaError_t launch_threshold_select(const float* gate, const int32_t* cu_seqlens, int nseq, int L, int max_len,
                                    const float* tau, int max_selected, int32_t* counts, int32_t* sel_idx,
                                    int32_t* cu_sel, uint32_t* status, cudaStream_t stream);

cudaError_t launch_threshold_update(const float* gate, const int32_t* cu_seqlens, int nseq, long long n_all,
                                    long long n_fixed, double ratio, float beta, float* tau, float* target_out,
                                    cudaStream_t stream);

// Decode step (decode.cu).
constexpr int kDecChunk = 512;  // cache positions per partial state
constexpr int kDecBlock = 16;   // cache positions per staged key/value block
struct DecodeParams {
    CUtensorMap tm_k, tm_v;     // caches as [B*Hkv][Lmax][d], box 64 x kDecBlock x 1, 128B swizzle
    const uint16_t *q, *k, *v;  // q [B, Hq, d]; caches [B, Hkv, Lmax, d]
    const int32_t* cache_len;   // [B]: the new token sits at cache_len - 1
    const float* gate;          // [B]
    const float* tau;           // one threshold (device)
    uint16_t* out;              // [B, Hq, d]
    int32_t* selected;          // [B] or nullptr
    float* part;                // partial states in the workspace
    uint32_t* status;           // workspace status word
    int B, Hq, Hkv, G, Lmax, d, W, chunk, nchunks;
    float scale_log2;
    unsigned long long timeout_ns;  // bound of every barrier wait
};
size_t decode_partials_bytes(int B, int Hkv, int G, int Lmax, int d);
cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream);

cudaError_t launch_attn(int mode, int d, const AttnParams& p, int max_seqlen, cudaStream_t stream);

// Backward pass (bwd.cu).
struct PrepParams {
    const uint16_t *q, *out, *dout;         // dense [B*Hq][L][d]
    const uint16_t *glob, *loc_sel;         // [Hq][sel_stride][d]: the two branches of selected rows
    const float* gate;                      // [B*L]
    const int32_t *cu_seqlens, *sel_idx, *cu_sel;
    float* dl;                              // D of the local rows [B*Hq][L]
    float* ds_sel;                          // D of the global rows [Hq][sel_stride]
    float* dgate;                           // [B*L]
    int32_t* slot;                          // [B*L]: row of the selection list, or -1
    uint16_t *q_sel, *do_sel;               // [Hq][sel_stride][d]: Q and sigmoid(g) dout of selected rows
    uint32_t* status;
    int B, Hq, L, nseq, sel_stride;
};

struct alignas(64) BwdParams {
    CUtensorMap tm_q, tm_do;    // dense [B*Hq][L][d]
    CUtensorMap tm_qs, tm_dos;  // selected rows [Hq][sel_stride][d]
    CUtensorMap tm_k, tm_v;     // [B*Hkv][L][d]
    const float *lse, *dl;      // [B*Hq][L]
    const float *lse_s, *ds_sel;  // [Hq][sel_stride]
    const int32_t *cu_seqlens, *sel_idx, *cu_sel, *slot;
    float* dq_sel;              // [Hq][sel_stride][d] fp32: global share of dQ
    uint16_t *dq, *dk, *dv;
    uint32_t* status;
    int Hq, Hkv, G, L, nseq, window, max_selected, sel_stride;
    float scale, scale_log2;
    unsigned long long timeout_ns;
};

cudaError_t launch_bwd_prep(const PrepParams& p, int d, cudaStream_t stream);
cudaError_t launch_bwd_dq(int mode, int d, const BwdParams& p, int max_seqlen, cudaStream_t stream);
cudaError_t launch_bwd_dkdv(int d, const BwdParams& p, int max_seqlen, cudaStream_t stream);
size_t bwd_smem_bytes(int d);

cudaError_t launch_timeout_probe(uint32_t* status, unsigned long long limit_ns, cudaStream_t stream);

size_t attn_smem_bytes(int d);

// Sets the text logo_last_error() returns on this host thread.
void set_last_error(const char* fmt, ...);

}  // namespace logo
