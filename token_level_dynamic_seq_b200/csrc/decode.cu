// Decode step: one new query token per sequence against its key/value cache,
// with the global branch read only for tokens whose gate passes the threshold.
//
// Sources: "Learning When to Attend", "Empirical Validation and System
// Optimization" (the savings carry over to time-to-first-token and token
// generation, the skipped work being memory-bound global reads);
// "LoGo: Token-Level Dynamic Local-Global Attention", Abstract (a gate decides
// per token, a threshold controller keeps the share).
//
// Memory-bound (about 4 FLOP per byte of cache read): the design goal is to
// keep enough cache bytes in flight and to spend few instructions per key.
//   decode_partial_kernel  persistent warps.  Work items are (512-position
//     chunk counted back from the new token, kv head, sequence); every warp
//     takes items round-robin on its own and skips, at the cost of a few
//     integer operations, the chunks before the window of a token that does
//     not take the global branch (the conditional global read).  A warp
//     streams its item's keys and values through a private ring of
//     kDecStages 16-position blocks in shared memory, filled by TMA
//     (128-byte swizzle) and tracked by one mbarrier per stage.  Per block:
//       S^T = K q^T   on the tensor cores (mma.sync m16n8k16, bf16 -> fp32):
//                     16 positions x 8 head columns (the G heads of the
//                     group, zero-padded), K fragments by ldmatrix;
//       online softmax per head in exp2 units (head columns sit in lanes,
//                     positions across lane groups: three shuffles per max);
//       O^T += V^T P^T  (mma.sync; V^T by ldmatrix.trans, P^T by movmatrix
//                     from the score fragment), O^T held in registers.
//     Each item writes two partial states (m, l, o) per head: over its
//     positions inside the window (local) and, for a selected token, over
//     all its positions (global).
//   decode_combine_kernel  grid (query head, sequence), one thread per output
//     column: merges the local partials of the window's chunks and, for a
//     selected token, the global partials of every chunk; then
//     o = local + sigmoid(g) * global, rounded once to bf16.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"

namespace logo {

namespace {

#ifndef LOGO_DEC_WARPS
#define LOGO_DEC_WARPS 4
#endif
#ifndef LOGO_DEC_STAGES
#define LOGO_DEC_STAGES 2
#endif
constexpr int kDecWarps = LOGO_DEC_WARPS;    // independent warps per CTA
constexpr int kDecStages = LOGO_DEC_STAGES;  // ring depth of each warp
constexpr int kDecThreads = 32 * kDecWarps;

__device__ __forceinline__ bool takes_global(float g, float tau) { return g > tau; }  // false for NaN

template <int D>
struct DecGeo {
    static constexpr int kBoxes = D / 64;                       // 64-column TMA boxes per row
    static constexpr int kBoxBytes = kDecBlock * 128;           // one box: 16 rows x 128 B
    static constexpr int kKVBytes = kBoxes * kBoxBytes;         // K (or V) of one block
    static constexpr int kStageBytes = 2 * kKVBytes;            // K then V
    static constexpr int kWarpBytes = kDecStages * kStageBytes;
    static constexpr int kSmemBytes = kDecWarps * kWarpBytes + 1024;  // + alignment slack
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ uint32_t movm_trans(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// D(16x8, fp32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Address of the 16-byte unit (row r, 8-column group u of a 64-column box) in a
// box written by TMA with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128(uint32_t box, int r, int u)
{
    return box + r * 128 + (((u ^ r) & 7) << 4);
}

// Online-softmax state of one warp for the (up to 8) heads of a group.  Lane
// (g, t) = (lane / 4, lane % 4) owns head columns 2t and 2t+1: their maxima
// (shared by the 8 lanes of the same t), a share of their sums, and O^T rows
// d = 16 mt + g and 16 mt + g + 8 of both heads.
template <int D>
struct DecState {
    float m[2], l[2];
    float o[D / 16][4];
    __device__ void init()
    {
        m[0] = m[1] = -INFINITY;
        l[0] = l[1] = 0.f;
        #pragma unroll
        for (int mt = 0; mt < D / 16; ++mt)
            #pragma unroll
            for (int e = 0; e < 4; ++e) o[mt][e] = 0.f;
    }
};

// Writes the warp's state (m, l, o[D]) for each real head of the group to
// `dst` ([G][D + 2] floats).
template <int D>
__device__ void store_state(const DecState<D>& st, int G, float* dst)
{
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    float l0 = st.l[0], l1 = st.l[1];
    #pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    #pragma unroll
    for (int c = 0; c < 2; ++c) {
        const int h = 2 * t + c;
        if (h >= G) continue;
        float* r = dst + h * (D + 2);
        if (g == 0) {
            r[0] = st.m[c];
            r[1] = c ? l1 : l0;
        }
        #pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            r[2 + 16 * mt + g] = st.o[mt][c];
            r[2 + 16 * mt + g + 8] = st.o[mt][2 + c];
        }
    }
}

// The ring of one warp: stage n % kDecStages holds block n of the warp's
// stream; `issued` and `used` count blocks over the warp's whole life, so the
// barrier parities carry across ranges and items.
struct Ring {
    uint32_t base;      // shared address of stage 0
    uint64_t* full;     // [kDecStages]
    int issued, used;
};

template <int D>
__device__ __forceinline__ void issue_block(const DecodeParams& p, Ring& ring, int row, int slab)
{
    using Geo = DecGeo<D>;
    const int s = ring.issued % kDecStages;
    uint8_t* dst = reinterpret_cast<uint8_t*>(__cvta_shared_to_generic(ring.base + s * Geo::kStageBytes));
    // The stage was last read by this warp's ldmatrix (generic proxy); order
    // those reads before the copy engine's writes.
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&ring.full[s], Geo::kStageBytes);
    #pragma unroll
    for (int bx = 0; bx < Geo::kBoxes; ++bx) {
        tma_load_3d(dst + bx * Geo::kBoxBytes, &p.tm_k, &ring.full[s], bx * 64, row, slab, policy_evict_first());
        tma_load_3d(dst + Geo::kKVBytes + bx * Geo::kBoxBytes, &p.tm_v, &ring.full[s], bx * 64, row, slab,
                    policy_evict_first());
    }
    ++ring.issued;
}

// Accumulates cache positions [a, e) of slab `slab` into the state; q
// fragments in bq.  Returns false when a wait ran out (the CTA aborts).
template <int D>
__device__ bool accumulate(const DecodeParams& p, Ring& ring, DecState<D>& st, const uint32_t (&bq)[D / 16][2],
                           int a, int e, int slab, volatile int* abort_flag)
{
    using Geo = DecGeo<D>;
    const int lane = threadIdx.x & 31, g = lane >> 2;
    const int nblk = (e - a + kDecBlock - 1) / kDecBlock;
    // prologue: up to kDecStages blocks in flight
    const int first = ring.issued;
    if (lane == 0)
        for (int i = 0; i < nblk && i < kDecStages; ++i) issue_block<D>(p, ring, a + i * kDecBlock, slab);
    ring.issued = first + (nblk < kDecStages ? nblk : kDecStages);
    const float sl2 = p.scale_log2;
    // ldmatrix lane roles: row within the 16-row block and 8-column group
    const int lr = (lane & 7) + 8 * ((lane >> 3) & 1);  // K: A rows (positions)
    const int lu = lane >> 4;                           // K: second 8 columns of the k-step
    const int vr = (lane & 7) + 8 * (lane >> 4);        // V (trans): positions
    const int vu = (lane >> 3) & 1;                     // V: second 8 columns (d) of the m-tile
    for (int i = 0; i < nblk; ++i) {
        const int s = ring.used % kDecStages;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&ring.full[s], (ring.used / kDecStages) & 1, abort_flag,
                                                          p.status, p.timeout_ns));
        if (!ok) return false;
        const uint32_t sK = ring.base + s * Geo::kStageBytes;
        const uint32_t sV = sK + Geo::kKVBytes;
        // S^T = K q^T: rows = positions g and g + 8, columns = heads 2t, 2t+1
        float c[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        #pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            uint32_t af[4];
            ldsm_x4(sw128(sK + (kk >> 2) * Geo::kBoxBytes, lr, 2 * (kk & 3) + lu), af);
            mma_bf16(c[kk & 1], af, bq[kk][0], bq[kk][1]);
        }
        const int k0 = a + i * kDecBlock;
        const bool v0 = k0 + g < e, v1 = k0 + g + 8 < e;
        float x[4];
        x[0] = v0 ? (c[0][0] + c[1][0]) * sl2 : -INFINITY;  // position g,     head 2t
        x[1] = v0 ? (c[0][1] + c[1][1]) * sl2 : -INFINITY;  // position g,     head 2t+1
        x[2] = v1 ? (c[0][2] + c[1][2]) * sl2 : -INFINITY;  // position g + 8, head 2t
        x[3] = v1 ? (c[0][3] + c[1][3]) * sl2 : -INFINITY;  // position g + 8, head 2t+1
        float bm0 = fmaxf(x[0], x[2]), bm1 = fmaxf(x[1], x[3]);
        #pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, off));
            bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, off));
        }
        const float mn0 = fmaxf(st.m[0], bm0), mn1 = fmaxf(st.m[1], bm1);
        const float r0 = mn0 == -INFINITY ? 0.f : mn0, r1 = mn1 == -INFINITY ? 0.f : mn1;
        const float al0 = fast_exp2(st.m[0] - r0), al1 = fast_exp2(st.m[1] - r1);  // 0 while empty
        st.m[0] = mn0;
        st.m[1] = mn1;
        const float p00 = fast_exp2(x[0] - r0), p01 = fast_exp2(x[1] - r1);
        const float p10 = fast_exp2(x[2] - r0), p11 = fast_exp2(x[3] - r1);
        st.l[0] = fmaf(st.l[0], al0, p00 + p10);
        st.l[1] = fmaf(st.l[1], al1, p01 + p11);
        #pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            st.o[mt][0] *= al0;
            st.o[mt][1] *= al1;
            st.o[mt][2] *= al0;
            st.o[mt][3] *= al1;
        }
        // P^T fragments: the score fragment's 8x8 halves transposed in registers
        const uint32_t pb0 = movm_trans(pack_bf16x2(p00, p01));  // positions 2t, 2t+1 of head g
        const uint32_t pb1 = movm_trans(pack_bf16x2(p10, p11));  // positions 2t+8, 2t+9
        // O^T += V^T P^T: rows d = 16 mt + g (+8), columns heads 2t, 2t+1
        #pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            uint32_t vf[4];
            ldsm_x4_trans(sw128(sV + (mt >> 2) * Geo::kBoxBytes, vr, 2 * (mt & 3) + vu), vf);
            mma_bf16(st.o[mt], vf, pb0, pb1);
        }
        ++ring.used;
        __syncwarp();
        if (lane == 0 && i + kDecStages < nblk) issue_block<D>(p, ring, a + (i + kDecStages) * kDecBlock, slab);
        ring.issued = ring.used + ((nblk - 1 - i) < kDecStages ? (nblk - 1 - i) : kDecStages);
    }
    return true;
}

template <int G, int D>
__global__ void __launch_bounds__(kDecThreads) decode_partial_kernel(const __grid_constant__ DecodeParams p)
{
    using Geo = DecGeo<D>;
    extern __shared__ uint8_t dsmem_raw[];
    __shared__ uint64_t full_bars[kDecWarps][kDecStages];
    __shared__ int abort_word;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;  // q fragment: head column g, d pairs 2t (+8)
    if (threadIdx.x == 0) abort_word = (*reinterpret_cast<volatile uint32_t*>(p.status) & kStatusTimeout) ? 1 : 0;
    if (lane == 0) {
        for (int s = 0; s < kDecStages; ++s) mbar_init(&full_bars[warp][s], 1);
        fence_barrier_init();
    }
    __syncthreads();
    volatile int* abort_flag = &abort_word;
    if (*abort_flag) return;
    if (lane == 0) {
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_v);
    }
    const uint32_t base = (smem_u32(dsmem_raw) + 1023u) & ~1023u;
    Ring ring{base + warp * Geo::kWarpBytes, full_bars[warp], 0, 0};
    const long long n_items = (long long)p.nchunks * p.Hkv * p.B;
    const long long stride = (long long)gridDim.x * kDecWarps;
    bool ok = true;
    for (long long it = (long long)blockIdx.x * kDecWarps + warp; it < n_items && ok; it += stride) {
        // Items run kv head fastest, then sequence, then chunk: the window chunks
        // of every token come first and every warp gets a similar mix.
        const int hk = (int)(it % p.Hkv);
        const long long bc = it / p.Hkv;
        const int b = (int)(bc % p.B), c = (int)(bc / p.B);
        const long long tpos = (long long)p.cache_len[b] - 1;
        if (tpos < 0) continue;
        if (tpos >= p.Lmax) {  // a cache length the cache cannot hold: reported, nothing read
            if (lane == 0 && c == 0 && hk == 0) atomicOr(p.status, kStatusBadArgument);
            continue;
        }
        const int hi = (int)(tpos + 1) - c * p.chunk;
        if (hi <= 0) continue;
        const int lo = hi - p.chunk > 0 ? hi - p.chunk : 0;
        const int wstart = (int)(tpos - p.W + 1 > 0 ? tpos - p.W + 1 : 0);
        const bool sel = takes_global(p.gate[b], *p.tau);
        const bool in_window = hi > wstart;
        if (!in_window && !sel) continue;  // keys outside the window are read only for the global branch
        // q^T fragments (B operand): column n = head g of the group, rows = d
        uint32_t bq[D / 16][2];
        const int gq = g < G ? g : 0;  // padding columns read nothing
        const uint32_t* qrow = reinterpret_cast<const uint32_t*>(p.q + ((long long)b * p.Hq + hk * G + gq) * D);
        #pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            bq[kk][0] = g < G ? __ldg(qrow + 8 * kk + t) : 0u;
            bq[kk][1] = g < G ? __ldg(qrow + 8 * kk + 4 + t) : 0u;
        }
        const int slab = b * p.Hkv + hk;
        float* part = p.part + (((long long)b * p.Hkv + hk) * p.nchunks + c) * 2 * G * (D + 2);
        DecState<D> st;
        st.init();
        const int mid = wstart < lo ? lo : (wstart > hi ? hi : wstart);
        // positions inside the window first ([mid, hi)): that state is the local partial
        if (in_window) {
            ok = accumulate<D>(p, ring, st, bq, mid, hi, slab, abort_flag);
            if (!ok) break;
            store_state<D>(st, G, part);
        }
        if (sel) {
            if (lo < mid) {
                ok = accumulate<D>(p, ring, st, bq, lo, mid, slab, abort_flag);
                if (!ok) break;
            }
            store_state<D>(st, G, part + G * (D + 2));  // global: all positions of the chunk
        }
    }
    if (!ok && lane == 0) {
        // Let every copy this warp started land before the CTA exits.
        volatile int dummy = 0;
        for (int n = ring.used; n < ring.issued; ++n)
            mbar_wait(&ring.full[n % kDecStages], (n / kDecStages) & 1, &dummy, nullptr, p.timeout_ns);
    }
    __syncwarp();
}

// One CTA per (sequence, query head): kDecCombineGroups groups of D threads,
// thread = output column; group k merges the chunks c = k (mod groups) and the
// groups' sums meet in shared memory.  The chunks' maximum is found by the
// whole block first, so every load of the sums is independent of the others
// (the loop is unrolled to keep several in flight).  One group: small CTAs,
// so the whole grid of B x Hq CTAs is resident at once.
#ifndef LOGO_DEC_COMBINE_GROUPS
#define LOGO_DEC_COMBINE_GROUPS 1
#endif
constexpr int kDecCombineGroups = LOGO_DEC_COMBINE_GROUPS;

__device__ __forceinline__ float block_max(float v, float* red)
{
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float m = -INFINITY;
    for (int w = 0; w < nw; ++w) m = fmaxf(m, red[w]);
    __syncthreads();  // red is reused
    return m;
}

template <int D>
__global__ void __launch_bounds__(kDecCombineGroups * D) decode_combine_kernel(const __grid_constant__ DecodeParams p)
{
    __shared__ float red_o[kDecCombineGroups][D];
    __shared__ float red_l[kDecCombineGroups];
    __shared__ float red_m[kDecCombineGroups * D / 32];
    const int h = blockIdx.x, b = blockIdx.y;
    const int col = threadIdx.x % D, grp = threadIdx.x / D;
    const int hk = h / p.G, gi = h % p.G;
    uint16_t* out = p.out + ((long long)b * p.Hq + h) * D;
    const long long t = (long long)p.cache_len[b] - 1;
    const float g = p.gate[b];
    const bool sel = takes_global(g, *p.tau);  // the gate's decision, whatever the cache holds
    if (p.selected && h == 0 && threadIdx.x == 0) p.selected[b] = sel ? 1 : 0;
    if (t < 0 || t >= p.Lmax) {
        if (grp == 0) out[col] = 0;
        return;
    }
    const long long wstart = t - p.W + 1 > 0 ? t - p.W + 1 : 0;
    const int n_chunks = (int)((t + p.chunk) / p.chunk);                 // ceil((t + 1) / chunk)
    const int n_local = (int)((t + 1 - wstart + p.chunk - 1) / p.chunk);  // chunks reaching into the window
    const float* base = p.part + ((long long)b * p.Hkv + hk) * p.nchunks * 2 * p.G * (D + 2);
    const long long kstride = 2LL * p.G * (D + 2);  // from one chunk's state to the next
    auto merge = [&](int kind, int n) {
        const float* st = base + (long long)kind * p.G * (D + 2) + gi * (D + 2);
        float mloc = -INFINITY;
        for (int c = threadIdx.x; c < n; c += blockDim.x) mloc = fmaxf(mloc, st[c * kstride]);
        const float M = block_max(mloc, red_m);
        float l = 0.f, o = 0.f;
        #pragma unroll 8
        for (int c = grp; c < n; c += kDecCombineGroups) {
            const float* r = st + c * kstride;
            const float m = r[0];
            const float f = (m == -INFINITY) ? 0.f : exp2f(m - M);
            l = fmaf(f, r[1], l);
            o = fmaf(f, r[2 + col], o);
        }
        red_o[grp][col] = o;
        if (col == 0) red_l[grp] = l;
        __syncthreads();
        float ot = 0.f, lt = 0.f;
        #pragma unroll
        for (int k = 0; k < kDecCombineGroups; ++k) {
            ot += red_o[k][col];
            lt += red_l[k];
        }
        __syncthreads();  // red_o and red_l are reused
        return lt > 0.f ? ot / lt : 0.f;
    };
    float val = merge(0, n_local);
    if (sel) {
        const float gs = 1.f / (1.f + expf(-g));
        val = fmaf(gs, merge(1, n_chunks), val);
    }
    if (grp == 0) {
        const __nv_bfloat16 r = __float2bfloat16_rn(val);
        out[col] = *reinterpret_cast<const uint16_t*>(&r);
    }
}

template <int G, int D>
cudaError_t launch_g_d(const DecodeParams& p, cudaStream_t stream)
{
    constexpr int smem = DecGeo<D>::kSmemBytes;
    auto kern = decode_partial_kernel<G, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDecThreads, smem)) != cudaSuccess) return e;
    const long long items = (long long)p.nchunks * p.Hkv * p.B;
    long long grid = (long long)sms * (per_sm > 0 ? per_sm : 1);
    const long long need = (items + kDecWarps - 1) / kDecWarps;
    if (grid > need) grid = need;
    if (grid < 1) grid = 1;
    kern<<<(unsigned)grid, kDecThreads, smem, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_combine_kernel<D><<<dim3(p.Hq, p.B), kDecCombineGroups * D, 0, stream>>>(p);
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
