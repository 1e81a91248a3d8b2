// Decode step: one new query token per sequence against its key/value cache,
// with the global branch read only for tokens whose gate passes the threshold.
//
// Sources: "Learning When to Attend", "Empirical Validation and System
// Optimization" (the savings carry over to time-to-first-token and token
// generation, the skipped work being memory-bound global reads);
// "LoGo: Token-Level Dynamic Local-Global Attention", Abstract (a gate decides
// per token, a threshold controller keeps the share).
//
// Memory-bound (about 4 FLOP per byte of cache read), so CUDA cores and
// coalesced loads rather than tensor cores.  Split over the cache:
//   decode_partial_kernel  grid (chunk, kv head, sequence); a CTA of 4 warps
//     takes kDecChunk keys, counted back from the new token.  Keys before the
//     window are read only when the token takes the global branch: for any
//     other token those CTAs exit at once (the conditional global read).  Per
//     32-key block a warp computes Q K^T with one key per lane (the G query
//     heads of the group from shared memory), an online softmax per head in
//     exp2 units, and P V with each lane owning d/32 output columns.  Each CTA
//     writes two partial states (m, l, o) per head: over its keys inside the
//     window (local) and over all its keys (global).
//   decode_combine_kernel  grid (query head, sequence), one thread per output
//     column: merges the local partials of the window's chunks and, for a
//     selected token, the global partials of every chunk; then
//     o = local + sigmoid(g) * global, rounded once to bf16.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"

namespace logo {

namespace {

constexpr int kDecWarps = 4;
constexpr int kDecThreads = 32 * kDecWarps;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ bool takes_global(float g, float tau) { return g > tau; }  // false for NaN

__device__ __forceinline__ float warp_max(float x)
{
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

__device__ __forceinline__ float warp_sum(float x)
{
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Online-softmax state of one warp for G heads; o holds D/32 columns per lane.
template <int G, int D>
struct WarpState {
    float m[G], l[G], o[G][D / 32];
    __device__ void init()
    {
        #pragma unroll
        for (int h = 0; h < G; ++h) {
            m[h] = -INFINITY;
            l[h] = 0.f;
            #pragma unroll
            for (int c = 0; c < D / 32; ++c) o[h][c] = 0.f;
        }
    }
};

// Accumulates keys [lo, hi) into the warp's state (the warp takes the 32-key
// blocks lo + 32 * warp, lo + 32 * (warp + kDecWarps), ...).
template <int G, int D>
__device__ void accumulate(WarpState<G, D>& st, const float* q_s, float* p_s, const uint16_t* kh, const uint16_t* vh,
                           long long lo, long long hi, float sl2)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (long long base = lo + 32LL * warp; base < hi; base += 32LL * kDecWarps) {
        const long long j = base + lane;
        const bool valid = j < hi;
        // Q K^T: one key per lane, its row read as 16-byte vectors.
        float s[G];
        #pragma unroll
        for (int h = 0; h < G; ++h) s[h] = 0.f;
        if (valid) {
            const uint4* kr = reinterpret_cast<const uint4*>(kh + j * D);
            #pragma unroll 4
            for (int c8 = 0; c8 < D / 8; ++c8) {
                const uint4 kv = __ldg(kr + c8);
                const uint32_t w4[4] = {kv.x, kv.y, kv.z, kv.w};
                #pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const float k0 = bf16_lo(w4[t]), k1 = bf16_hi(w4[t]);
                    #pragma unroll
                    for (int h = 0; h < G; ++h) {
                        s[h] = fmaf(q_s[h * D + c8 * 8 + 2 * t], k0, s[h]);
                        s[h] = fmaf(q_s[h * D + c8 * 8 + 2 * t + 1], k1, s[h]);
                    }
                }
            }
        }
        // Online softmax per head (exp2 units).
        #pragma unroll
        for (int h = 0; h < G; ++h) {
            const float x = valid ? s[h] * sl2 : -INFINITY;
            const float m_new = fmaxf(st.m[h], warp_max(x));
            const float alpha = (st.m[h] == -INFINITY) ? 0.f : exp2f(st.m[h] - m_new);
            const float p = valid ? exp2f(x - m_new) : 0.f;
            st.l[h] = st.l[h] * alpha + warp_sum(p);
            #pragma unroll
            for (int c = 0; c < D / 32; ++c) st.o[h][c] *= alpha;
            st.m[h] = m_new;
            p_s[(warp * G + h) * 32 + lane] = p;
        }
        __syncwarp();
        // P V: lane owns columns lane * D/32 .. ; one value row per key, coalesced.
        const int nk = (int)min(32LL, hi - base);
        for (int jj = 0; jj < nk; ++jj) {
            const uint16_t* vr = vh + (base + jj) * D + lane * (D / 32);
            float vv[D / 32];
            if constexpr (D == 128) {
                const uint2 w = __ldg(reinterpret_cast<const uint2*>(vr));
                vv[0] = bf16_lo(w.x);
                vv[1] = bf16_hi(w.x);
                vv[2] = bf16_lo(w.y);
                vv[3] = bf16_hi(w.y);
            } else {
                const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(vr));
                vv[0] = bf16_lo(w);
                vv[1] = bf16_hi(w);
            }
            #pragma unroll
            for (int h = 0; h < G; ++h) {
                const float p = p_s[(warp * G + h) * 32 + jj];
                #pragma unroll
                for (int c = 0; c < D / 32; ++c) st.o[h][c] = fmaf(p, vv[c], st.o[h][c]);
            }
        }
        __syncwarp();
    }
}

// Merges the warps' states and writes (m, l, o[D]) per head to `dst` (stride D + 2).
template <int G, int D>
__device__ void store_partial(const WarpState<G, D>& st, float* red, float* dst)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // red: [kDecWarps][G][D + 2]
    #pragma unroll
    for (int h = 0; h < G; ++h) {
        float* r = red + (warp * G + h) * (D + 2);
        if (lane == 0) {
            r[0] = st.m[h];
            r[1] = st.l[h];
        }
        #pragma unroll
        for (int c = 0; c < D / 32; ++c) r[2 + lane * (D / 32) + c] = st.o[h][c];
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * D; idx += kDecThreads) {
        const int h = idx / D, c = idx % D;
        float M = -INFINITY;
        #pragma unroll
        for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, red[(w * G + h) * (D + 2)]);
        float l = 0.f, o = 0.f;
        #pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
            const float* r = red + (w * G + h) * (D + 2);
            const float f = (r[0] == -INFINITY) ? 0.f : exp2f(r[0] - M);
            l += f * r[1];
            o += f * r[2 + c];
        }
        float* out = dst + h * (D + 2);
        if (c == 0) {
            out[0] = M;
            out[1] = l;
        }
        out[2 + c] = o;
    }
    __syncthreads();
}

template <int G, int D>
__global__ void __launch_bounds__(kDecThreads) decode_partial_kernel(DecodeParams p)
{
    __shared__ float q_s[G * D];
    __shared__ float p_s[kDecWarps * G * 32];
    __shared__ float red[kDecWarps * G * (D + 2)];
    const int c = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const long long t = (long long)p.cache_len[b] - 1;
    if (t < 0) return;
    if (t >= p.Lmax) {  // a cache length the cache cannot hold: reported, nothing read
        if (threadIdx.x == 0 && c == 0 && hk == 0) atomicOr(p.status, kStatusBadArgument);
        return;
    }
    const long long hi = t + 1 - (long long)c * p.chunk;
    if (hi <= 0) return;
    const long long lo = hi - p.chunk > 0 ? hi - p.chunk : 0;
    const long long wstart = t - p.W + 1 > 0 ? t - p.W + 1 : 0;
    const bool sel = takes_global(p.gate[b], *p.tau);
    const bool in_window = hi > wstart;
    if (!in_window && !sel) return;  // keys outside the window are read only for the global branch

    for (int i = threadIdx.x; i < G * D; i += kDecThreads) {
        const int h = i / D, cc = i % D;
        const uint16_t qb = p.q[((long long)b * p.Hq + hk * G + h) * D + cc];
        q_s[i] = __uint_as_float((uint32_t)qb << 16);
    }
    __syncthreads();
    const uint16_t* kh = p.k + ((long long)b * p.Hkv + hk) * (long long)p.Lmax * D;
    const uint16_t* vh = p.v + ((long long)b * p.Hkv + hk) * (long long)p.Lmax * D;
    float* part = p.part + (((long long)b * p.Hkv + hk) * p.nchunks + c) * 2 * G * (D + 2);

    WarpState<G, D> st;
    st.init();
    // keys inside the window first ([mid, hi)): that state is the local partial
    const long long mid = wstart < lo ? lo : (wstart > hi ? hi : wstart);
    if (in_window) accumulate<G, D>(st, q_s, p_s, kh, vh, mid, hi, p.scale_log2);
    store_partial<G, D>(st, red, part);  // local (empty if the chunk is outside the window)
    if (sel) {
        if (lo < mid) accumulate<G, D>(st, q_s, p_s, kh, vh, lo, mid, p.scale_log2);
        store_partial<G, D>(st, red, part + G * (D + 2));  // global: all keys of the chunk
    }
}

// One thread per output column of one (sequence, query head).
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(DecodeParams p)
{
    const int h = blockIdx.x, b = blockIdx.y, col = threadIdx.x;
    const int hk = h / p.G, gi = h % p.G;
    uint16_t* out = p.out + ((long long)b * p.Hq + h) * D;
    const long long t = (long long)p.cache_len[b] - 1;
    const float g = p.gate[b];
    const bool sel = takes_global(g, *p.tau);  // the gate's decision, whatever the cache holds
    if (p.selected && h == 0 && col == 0) p.selected[b] = sel ? 1 : 0;
    if (t < 0 || t >= p.Lmax) {
        out[col] = 0;
        return;
    }
    const long long wstart = t - p.W + 1 > 0 ? t - p.W + 1 : 0;
    const int n_chunks = (int)((t + p.chunk) / p.chunk);                 // ceil((t + 1) / chunk)
    const int n_local = (int)((t + 1 - wstart + p.chunk - 1) / p.chunk);  // chunks reaching into the window
    const float* base = p.part + ((long long)b * p.Hkv + hk) * p.nchunks * 2 * p.G * (D + 2);
    auto merge = [&](int kind, int n) {
        float M = -INFINITY;
        for (int c = 0; c < n; ++c) M = fmaxf(M, base[((long long)c * 2 + kind) * p.G * (D + 2) + gi * (D + 2)]);
        float l = 0.f, o = 0.f;
        for (int c = 0; c < n; ++c) {
            const float* r = base + ((long long)c * 2 + kind) * p.G * (D + 2) + gi * (D + 2);
            const float f = (r[0] == -INFINITY) ? 0.f : exp2f(r[0] - M);
            l += f * r[1];
            o += f * r[2 + col];
        }
        return l > 0.f ? o / l : 0.f;
    };
    float val = merge(0, n_local);
    if (sel) {
        const float gs = 1.f / (1.f + expf(-g));
        val = fmaf(gs, merge(1, n_chunks), val);
    }
    const __nv_bfloat16 r = __float2bfloat16_rn(val);
    out[col] = *reinterpret_cast<const uint16_t*>(&r);
}

template <int G, int D>
cudaError_t launch_g_d(const DecodeParams& p, cudaStream_t stream)
{
    dim3 grid(p.nchunks, p.Hkv, p.B);
    decode_partial_kernel<G, D><<<grid, kDecThreads, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_combine_kernel<D><<<dim3(p.Hq, p.B), D, 0, stream>>>(p);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const DecodeParams& p, cudaStream_t stream)
{
    switch (p.G) {
        case 1: return launch_g_d<1, D>(p, stream);
        case 2: return launch_g_d<2, D>(p, stream);
        case 4: return launch_g_d<4, D>(p, stream);
        case 8: return launch_g_d<8, D>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

size_t decode_partials_bytes(int B, int Hkv, int G, int Lmax, int d)
{
    const long long nchunks = (Lmax + kDecChunk - 1) / kDecChunk;
    return (size_t)B * Hkv * (size_t)(nchunks > 0 ? nchunks : 1) * 2 * G * (d + 2) * sizeof(float);
}

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream)
{
    if (p.B == 0) return cudaSuccess;
    return p.d == 64 ? launch_d<64>(p, stream) : launch_d<128>(p, stream);
}

}  // namespace logo
