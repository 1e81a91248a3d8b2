// Budget rule on the GPU: per sequence, the k = budget_count(ratio, len)
// positions with the largest gate logits, ties to the lower position, emitted
// in ascending order.
//
// Sources: "LoGo: Token-Level Dynamic Local-Global Attention", Abstract (a
// gate decides per token whether the global branch runs; the share of such
// tokens is held at a set value); "Learning When to Attend", "The
// Architecture of Conditional Attention" (a yes/no routing decision for each
// position, about one in five going global).
//
// Each sequence is spread over a cluster of up to kClusterCtas CTAs (one CTA per 4096 tokens
// of the longest sequence, rounded up to a power of two), CTA r holding the r-th contiguous
// slice of the sequence:
//  1. map each fp32 logit to a 32-bit key whose unsigned order is the
//     selection order (-0 folded onto +0, every NaN to 0, below -inf); a slice
//     of up to kSliceResident keys stays in shared memory for every later pass,
//     a longer one is re-read from the logits each pass;
//  2. radix-select the k-th largest key T with four 8-bit passes: each CTA
//     counts its slice into a shared-memory histogram, and after a cluster
//     barrier every CTA sums the cluster's histograms through distributed
//     shared memory and takes the same digit; the last pass also gives how
//     many keys equal to T there are, and how many of them must be taken;
//  3. stream-compact in ascending position order: each CTA's keys above T and
//     equal to T are counted and exchanged the same way, so a slice's selected
//     positions go after those of the lower-ranked slices, and the keys equal to
//     T are taken lowest position first up to the count.
// The threshold form (further down) counts and compacts the positions above a
// threshold on the same clusters, and its controller step finds one order
// statistic of the whole batch with the same radix passes.
// Integer work only, so the result is bit-exact.
#include <cuda_runtime.h>

#include <cstdint>
#include <utility>

#include "kernels.cuh"

namespace logo {

namespace {

constexpr int kItems = 4;

__device__ __forceinline__ uint32_t gate_key(float f)
{
    uint32_t b = __float_as_uint(f);
    if ((b & 0x7FFFFFFFu) > 0x7F800000u) return 0u;  // NaN ranks below everything
    if (b == 0x80000000u) b = 0u;                      // -0 equals +0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// ---------------------------------------------------------------- cluster form
//
// The top-k selection: each sequence spread over a cluster of up to kClusterCtas CTAs, CTA r of
// the cluster holding the r-th contiguous slice of the sequence's keys.  Every radix pass counts
// the slice into a CTA histogram, one cluster barrier later each CTA sums all the cluster's
// histograms through distributed shared memory and takes the same digit; the compaction places
// each CTA's slice after the selected keys of the lower-ranked slices (their counts are read the
// same way), so positions still come out ascending and ties still go to the lower position.
// Every CTA of a cluster works on the same sequence and takes the same branches, so all of them
// reach every cluster barrier.

constexpr int kClusterCtas = 8;        // largest cluster
constexpr int kKeysPerCta = 4096;      // a cluster gets one CTA per this many keys (power of two)
constexpr int kCThreads = 512;
constexpr int kCWarps = kCThreads / 32;
constexpr int kSliceResident = 40960;  // keys of one slice kept in shared memory (160 KB)

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_nctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of the same shared-memory variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(const void* local, uint32_t rank)
{
    uint32_t a = (uint32_t)__cvta_generic_to_shared(local), r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ long long ld_cluster_s64(uint32_t addr)
{
    long long v;
    asm volatile("ld.shared::cluster.s64 %0, [%1];" : "=l"(v) : "r"(addr) : "memory");
    return v;
}

// Exclusive prefix sum over a kCThreads block; `total` receives the block sum.
__device__ __forceinline__ int cblock_exclusive_scan(int v, int* warp_buf, int& total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_buf[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int s = lane < kCWarps ? warp_buf[lane] : 0;
        #pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < kCWarps) warp_buf[lane] = s;  // inclusive
    }
    __syncthreads();
    const int before = warp ? warp_buf[warp - 1] : 0;
    total = warp_buf[kCWarps - 1];
    __syncthreads();  // warp_buf may be reused right after
    return before + x - v;
}

struct ClusterKth {
    uint32_t key;        // the k-th largest key of the cluster's keys
    long long take_eq;   // how many keys equal to it are among the k largest
    long long eq_count;  // how many keys equal to it there are
};

// Radix select over the keys of all CTAs of the cluster (this CTA's slice: key_at(i), i < n)
// with four 8-bit passes, 1 <= k <= the cluster's key count.  Called by every thread of every
// CTA of the cluster with the same k.  Each pass counts the slice into a shared-memory
// histogram; after a cluster barrier every CTA sums the cluster's histograms through
// distributed shared memory and takes the same digit.  The caller passes one more cluster
// barrier before its CTA exits, so no CTA leaves while another still reads its histograms.
template <typename KeyAt>
__device__ ClusterKth cluster_kth_largest(KeyAt key_at, long long n, long long k, uint32_t nranks)
{
    __shared__ uint32_t hist[2][256];  // this slice's counts, alternating between passes
    __shared__ uint32_t tot[256];      // the cluster's counts
    __shared__ uint32_t sh_digit, sh_bin_count;
    __shared__ long long sh_remaining;
    const int tid = threadIdx.x;
    uint32_t prefix = 0, mask = 0;
    long long remaining = k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass, b = pass & 1;
        if (tid < 256) hist[b][tid] = 0;
        __syncthreads();
        for (long long i = tid; i < n; i += kCThreads) {
            const uint32_t key = key_at(i);
            if ((key & mask) == prefix) atomicAdd(&hist[b][(key >> shift) & 255u], 1u);
        }
        // Every slice's counts of this pass are complete.  A CTA writes hist[b] again two
        // passes later, after the next barrier, which no CTA passes before it has read these.
        cluster_sync_all();
        if (tid < 256) {
            uint32_t c = 0;
            for (uint32_t r = 0; r < nranks; ++r) c += ld_cluster_u32(cluster_map(&hist[b][tid], r));
            tot[tid] = c;
        }
        __syncthreads();
        if (tid < 32) {
            // lane l owns bins 255-8l .. 248-8l (descending)
            const int lane = tid;
            uint32_t c[8];
            uint32_t sum = 0;
            #pragma unroll
            for (int t = 0; t < 8; ++t) {
                c[t] = tot[255 - 8 * lane - t];
                sum += c[t];
            }
            uint32_t incl = sum;
            #pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const long long excl = (long long)(incl - sum);
            if (excl < remaining && remaining <= excl + (long long)sum) {
                long long acc = excl;
                #pragma unroll
                for (int t = 0; t < 8; ++t) {
                    if (acc + (long long)c[t] >= remaining) {
                        sh_digit = 255u - 8u * lane - t;
                        sh_remaining = remaining - acc;
                        sh_bin_count = c[t];
                        break;
                    }
                    acc += c[t];
                }
            }
        }
        __syncthreads();
        prefix |= sh_digit << shift;
        mask |= 255u << shift;
        remaining = sh_remaining;
    }
    ClusterKth r;
    r.key = prefix;
    r.take_eq = remaining;
    r.eq_count = (long long)sh_bin_count;
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(kCThreads)
    select_cluster_kernel(const float* __restrict__ gate, const int32_t* __restrict__ cu_seqlens, int nseq, int L,
                          double ratio, int32_t* __restrict__ sel_idx, int32_t* __restrict__ cu_sel, int resident_cap)
{
    extern __shared__ uint32_t slice_keys[];  // resident_cap keys (at most kSliceResident)
    __shared__ long long cnt[2];              // keys of this slice above T, equal to T
    __shared__ int warp_buf[32];
    __shared__ long long sh_sel_before, sh_eq_quota;

    const uint32_t rank = cluster_ctarank();
    const uint32_t nranks = cluster_nctarank();  // the launch's cluster size, 1 to kClusterCtas
    const int s = blockIdx.y;
    const int tid = threadIdx.x;
    long long start, len, out_off;
    if (cu_seqlens) {
        start = cu_seqlens[s];
        len = (long long)cu_seqlens[s + 1] - start;
        out_off = 0;
        for (int t = 0; t < s; ++t) out_off += budget_count(ratio, (long long)cu_seqlens[t + 1] - cu_seqlens[t]);
    } else {
        start = (long long)s * L;
        len = L;
        out_off = (long long)s * budget_count(ratio, L);
    }
    const long long k = budget_count(ratio, len);  // the same in every CTA of the cluster
    if (rank == 0 && tid == 0) {
        cu_sel[s + 1] = (int32_t)(out_off + k);
        if (s == 0) cu_sel[0] = 0;
    }
    if (k <= 0) return;
    const long long lo = len * rank / nranks, hi = len * (rank + 1) / nranks, n = hi - lo;
    const float* g = gate + start + lo;
    int32_t* out = sel_idx + out_off;
    if (k == len) {
        for (long long i = tid; i < n; i += kCThreads) out[lo + i] = (int32_t)(lo + i);
        return;
    }
    const bool resident = n <= resident_cap;  // the launch sized the array for the longest sequence
    if (resident)
        for (long long i = tid; i < n; i += kCThreads) slice_keys[i] = gate_key(__ldg(g + i));
    auto key_at = [&](long long i) -> uint32_t { return resident ? slice_keys[i] : gate_key(__ldg(g + i)); };

    // ---- radix select of the k-th largest key over the whole sequence
    const ClusterKth kr = cluster_kth_largest(key_at, n, k, nranks);
    const uint32_t T = kr.key;                    // the k-th largest key
    const long long take_eq = kr.take_eq;         // how many keys equal to T are selected
    const bool all_eq = take_eq == kr.eq_count;

    // ---- this slice's keys above and equal to T, then its place among the cluster's slices
    int n_gt = 0, n_eq = 0;
    for (long long i = tid; i < n; i += kCThreads) {
        const uint32_t key = key_at(i);
        n_gt += key > T ? 1 : 0;
        n_eq += key == T ? 1 : 0;
    }
    int tot_gt, tot_eq;
    cblock_exclusive_scan(n_gt, warp_buf, tot_gt);
    cblock_exclusive_scan(n_eq, warp_buf, tot_eq);
    if (tid == 0) {
        cnt[0] = tot_gt;
        cnt[1] = tot_eq;
    }
    cluster_sync_all();
    if (tid == 0) {
        long long gt_before = 0, eq_before = 0;
        for (uint32_t r = 0; r < rank; ++r) {
            gt_before += ld_cluster_s64(cluster_map(&cnt[0], r));
            eq_before += ld_cluster_s64(cluster_map(&cnt[1], r));
        }
        const long long eq_taken_before = all_eq ? eq_before : (eq_before < take_eq ? eq_before : take_eq);
        sh_sel_before = gt_before + eq_taken_before;
        const long long q = all_eq ? (long long)tot_eq : take_eq - eq_taken_before;
        sh_eq_quota = q < 0 ? 0 : (q > tot_eq ? tot_eq : q);
    }
    __syncthreads();
    const long long eq_quota = sh_eq_quota;
    const bool take_all_eq = eq_quota == (long long)tot_eq;

    // ---- compaction of the slice in ascending position order
    long long eq_seen = 0, written = sh_sel_before;
    for (long long chunk = 0; chunk < n; chunk += (long long)kCThreads * kItems) {
        const long long i0 = chunk + (long long)tid * kItems;
        uint32_t keys[kItems];
        int n_eq_t = 0;
        #pragma unroll
        for (int t = 0; t < kItems; ++t) {
            keys[t] = (i0 + t < n) ? key_at(i0 + t) : 0u;
            n_eq_t += (i0 + t < n && keys[t] == T) ? 1 : 0;
        }
        int eq_total = 0, eq_before = 0;
        if (!take_all_eq) eq_before = cblock_exclusive_scan(n_eq_t, warp_buf, eq_total);
        bool sel[kItems];
        int n_sel = 0, eq_run = 0;
        #pragma unroll
        for (int t = 0; t < kItems; ++t) {
            const bool in = i0 + t < n;
            const bool gt = in && keys[t] > T;
            const bool eq = in && keys[t] == T;
            sel[t] = gt || (eq && (take_all_eq || (eq_seen + eq_before + eq_run) < eq_quota));
            eq_run += eq ? 1 : 0;
            n_sel += sel[t] ? 1 : 0;
        }
        int sel_total;
        const int sel_before = cblock_exclusive_scan(n_sel, warp_buf, sel_total);
        int o = 0;
        #pragma unroll
        for (int t = 0; t < kItems; ++t)
            if (sel[t]) out[written + sel_before + (o++)] = (int32_t)(lo + i0 + t);
        eq_seen += eq_total;
        written += sel_total;
    }
    // No CTA leaves while another may still read its shared memory.
    cluster_sync_all();
}

// ---------------------------------------------------------------- threshold form
//
// "LoGo: Token-Level Dynamic Local-Global Attention", Abstract: the budget is
// kept by a controller that moves a threshold on the gate.  A token takes the
// global branch iff its logit is strictly above the threshold (never for a NaN
// logit or a NaN threshold); the comparison is done on the order-preserving
// keys, so it is exact (-0 equals +0, no flushing of subnormals).

__device__ __forceinline__ bool above(uint32_t gkey, uint32_t tkey, bool tau_nan)
{
    return !tau_nan && gkey > tkey;
}

__device__ __forceinline__ void seq_span(const int32_t* cu_seqlens, int L, int s, long long& start, long long& len)
{
    if (cu_seqlens) {
        start = cu_seqlens[s];
        len = (long long)cu_seqlens[s + 1] - start;
    } else {
        start = (long long)s * L;
        len = L;
    }
}

__device__ __forceinline__ float key_to_float(uint32_t key)
{
    if (key == 0u) return __int_as_float(0x7fc00000);  // NaN
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// The threshold rule and the controller step on clusters of CTAs: a sequence (for the
// controller, the whole batch) in contiguous slices exactly as in the top-k selection above.

// Slice count of logits above the threshold, summed over the cluster into counts[s].
__global__ void __launch_bounds__(kCThreads) threshold_count_cluster_kernel(const float* __restrict__ gate,
                                                                           const int32_t* __restrict__ cu_seqlens,
                                                                           int L, const float* __restrict__ tau,
                                                                           int32_t* __restrict__ counts)
{
    __shared__ int warp_buf[32];
    __shared__ long long slice_count;
    const uint32_t rank = cluster_ctarank(), nranks = cluster_nctarank();
    const int s = blockIdx.y;
    long long start, len;
    seq_span(cu_seqlens, L, s, start, len);
    const long long lo = len * rank / nranks, hi = len * (rank + 1) / nranks;
    const float t = *tau;
    const bool tau_nan = isnan(t);
    const uint32_t tkey = gate_key(t);
    int c = 0;
    for (long long i = lo + threadIdx.x; i < hi; i += kCThreads) c += above(gate_key(__ldg(gate + start + i)), tkey, tau_nan);
    int total;
    cblock_exclusive_scan(c, warp_buf, total);
    if (threadIdx.x == 0) slice_count = total;
    cluster_sync_all();
    if (rank == 0 && threadIdx.x == 0) {
        long long sum = 0;
        for (uint32_t r = 0; r < nranks; ++r) sum += ld_cluster_s64(cluster_map(&slice_count, r));
        counts[s] = (int32_t)sum;
    }
    cluster_sync_all();  // no CTA leaves while rank 0 still reads its count
}

// Per sequence: the positions above the threshold, ascending, at most `cap` of them, written at
// the sequence's offset (the capped counts of the earlier sequences); each slice after the
// positions of the lower-ranked slices.
__global__ void __launch_bounds__(kCThreads) threshold_compact_cluster_kernel(
    const float* __restrict__ gate, const int32_t* __restrict__ cu_seqlens, int L, const float* __restrict__ tau,
    int cap, const int32_t* __restrict__ counts, int32_t* __restrict__ sel_idx, int32_t* __restrict__ cu_sel,
    uint32_t* status)
{
    __shared__ int warp_buf[32];
    __shared__ long long slice_count, sh_before;
    const uint32_t rank = cluster_ctarank(), nranks = cluster_nctarank();
    const int s = blockIdx.y;
    long long start, len;
    seq_span(cu_seqlens, L, s, start, len);
    long long off = 0;
    for (int t = 0; t < s; ++t) off += min(counts[t], cap);
    const int mine = min(counts[s], cap);
    if (rank == 0 && threadIdx.x == 0) {
        cu_sel[s + 1] = (int32_t)(off + mine);
        if (s == 0) cu_sel[0] = 0;
        if (counts[s] > cap) atomicOr(status, kStatusCapacity);
    }
    if (mine == 0) return;  // the same in every CTA of the cluster
    const long long lo = len * rank / nranks, hi = len * (rank + 1) / nranks;
    const float t = *tau;
    const bool tau_nan = isnan(t);
    const uint32_t tkey = gate_key(t);
    int c = 0;
    for (long long i = lo + threadIdx.x; i < hi; i += kCThreads) c += above(gate_key(__ldg(gate + start + i)), tkey, tau_nan);
    int total;
    cblock_exclusive_scan(c, warp_buf, total);
    if (threadIdx.x == 0) slice_count = total;
    cluster_sync_all();
    if (threadIdx.x == 0) {
        long long before = 0;
        for (uint32_t r = 0; r < rank; ++r) before += ld_cluster_s64(cluster_map(&slice_count, r));
        sh_before = before;
    }
    __syncthreads();
    int32_t* out = sel_idx + off;
    long long written = sh_before;
    for (long long chunk = lo; chunk < hi && written < mine; chunk += (long long)kCThreads * kItems) {
        const long long i0 = chunk + (long long)threadIdx.x * kItems;
        bool sel[kItems];
        int n_sel = 0;
        #pragma unroll
        for (int u = 0; u < kItems; ++u) {
            sel[u] = (i0 + u < hi) && above(gate_key(__ldg(gate + start + i0 + u)), tkey, tau_nan);
            n_sel += sel[u] ? 1 : 0;
        }
        int chunk_total;
        const int before = cblock_exclusive_scan(n_sel, warp_buf, chunk_total);
        int o = 0;
        #pragma unroll
        for (int u = 0; u < kItems; ++u) {
            if (sel[u]) {
                const long long dst = written + before + (o++);
                if (dst < mine) out[dst] = (int32_t)(i0 + u);
            }
        }
        written += chunk_total;
    }
    cluster_sync_all();  // no CTA leaves while a higher rank still reads its count
}

// The controller step over the whole batch (all n valid logits): target q = the (k+1)-th
// largest logit, k = budget_count(ratio, n) (-inf when k = n, or when that place holds a NaN);
// tau <- tau + beta * (q - tau) in fp32 with a rounding after each operation, or tau <- q when
// either is not finite.  The batch is spread over the cluster in contiguous slices.
__global__ void __launch_bounds__(kCThreads) threshold_update_cluster_kernel(
    const float* __restrict__ gate, const int32_t* __restrict__ cu_seqlens, int nseq, long long n_fixed, double ratio,
    float beta, float* __restrict__ tau, float* __restrict__ target_out, int resident_cap)
{
    extern __shared__ uint32_t slice_keys[];  // resident_cap keys
    const uint32_t rank = cluster_ctarank(), nranks = cluster_nctarank();
    const long long n_all = cu_seqlens ? (long long)cu_seqlens[nseq] : n_fixed;
    const long long k = budget_count(ratio, n_all);
    float q = -INFINITY;
    if (k < n_all) {  // the same in every CTA of the cluster
        const long long lo = n_all * rank / nranks, hi = n_all * (rank + 1) / nranks, n = hi - lo;
        const float* g = gate + lo;
        const bool resident = n <= resident_cap;
        if (resident)
            for (long long i = threadIdx.x; i < n; i += kCThreads) slice_keys[i] = gate_key(__ldg(g + i));
        auto key_at = [&](long long i) -> uint32_t { return resident ? slice_keys[i] : gate_key(__ldg(g + i)); };
        const ClusterKth r = cluster_kth_largest(key_at, n, k + 1, nranks);
        q = key_to_float(r.key);
        if (isnan(q)) q = -INFINITY;
        cluster_sync_all();  // no CTA leaves while another still reads its histograms
    }
    if (rank == 0 && threadIdx.x == 0) {
        const float t = *tau;
        const bool finite = isfinite(t) && isfinite(q);
        *tau = finite ? __fadd_rn(t, __fmul_rn(beta, __fsub_rn(q, t))) : q;
        if (target_out) *target_out = q;
    }
}

// CTAs per cluster for `n` keys: one per kKeysPerCta, a power of two, at most kClusterCtas.
int cluster_ctas_for(long long n)
{
    int ctas = 1;
    while (ctas < kClusterCtas && (long long)ctas * kKeysPerCta < n) ctas *= 2;
    return ctas;
}

template <typename... Args, typename... Act>
cudaError_t launch_cluster(void (*kern)(Args...), int ctas, int nseq, size_t smem, cudaStream_t stream, Act&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ctas, nseq);
    cfg.blockDim = dim3(kCThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ctas;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Act>(args)...);
}

}  // namespace

cudaError_t launch_threshold_select(const float* gate, const int32_t* cu_seqlens, int nseq, int L, int max_len,
                                    const float* tau, int max_selected, int32_t* counts, int32_t* sel_idx,
                                    int32_t* cu_sel, uint32_t* status, cudaStream_t stream)
{
    if (nseq <= 0) return cudaSuccess;
    const int ctas = cluster_ctas_for(max_len > 0 ? max_len : 1);
    cudaError_t e = launch_cluster(threshold_count_cluster_kernel, ctas, nseq, 0, stream, gate, cu_seqlens, L, tau,
                                   counts);
    if (e != cudaSuccess) return e;
    return launch_cluster(threshold_compact_cluster_kernel, ctas, nseq, 0, stream, gate, cu_seqlens, L, tau,
                          max_selected, (const int32_t*)counts, sel_idx, cu_sel, status);
}

cudaError_t launch_threshold_update(const float* gate, const int32_t* cu_seqlens, int nseq, long long n_all,
                                    long long n_fixed, double ratio, float beta, float* tau, float* target_out,
                                    cudaStream_t stream)
{
    // n_all: the number of logits of the batch as the host knows it (B * L, or the packed
    // total), which sizes the cluster; the kernel reads the packed total from cu_seqlens.
    const int ctas = cluster_ctas_for(n_all > 0 ? n_all : 1);
    const long long slice = ((n_all > 0 ? n_all : 1) + ctas - 1) / ctas;
    const int cap = (int)(slice < kSliceResident ? slice : kSliceResident);
    const size_t smem = (size_t)cap * 4;
    cudaError_t e =
        cudaFuncSetAttribute(threshold_update_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_cluster(threshold_update_cluster_kernel, ctas, 1, smem, stream, gate, cu_seqlens, nseq, n_fixed,
                          ratio, beta, tau, target_out, cap);
}

cudaError_t launch_select(const float* gate, const int32_t* cu_seqlens, int nseq, int L, int max_len,
                          double ratio, int32_t* sel_idx, int32_t* cu_sel, cudaStream_t stream)
{
    if (nseq <= 0) return cudaSuccess;
    // One cluster per sequence, of one CTA per kKeysPerCta keys of the longest sequence (a power
    // of two, at most kClusterCtas); its slices of at most kSliceResident keys stay in shared
    // memory.
    const long long ml = max_len > 0 ? max_len : 1;
    const int ctas = cluster_ctas_for(ml);
    const long long slice = (ml + ctas - 1) / ctas;
    const int cap = (int)(slice < kSliceResident ? slice : kSliceResident);
    const size_t smem = (size_t)cap * 4;
    cudaError_t e = cudaFuncSetAttribute(select_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_cluster(select_cluster_kernel, ctas, nseq, smem, stream, gate, cu_seqlens, nseq, L, ratio, sel_idx,
                          cu_sel, cap);
}

}  // namespace logo
