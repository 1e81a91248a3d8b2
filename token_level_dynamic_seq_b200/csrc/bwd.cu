// Backward pass of local + selected-query global attention for sm_100a.
//
// Method sources (page titles and sections): "LoGo: Token-Level Dynamic
// Local-Global Attention", Abstract (a learned gate trained with the model, no
// auxiliary loss; kernels that skip the global work of unselected queries);
// "Learning When to Attend", "Empirical Validation and System Optimization"
// (trained end to end; the speed-up is claimed for training throughput).  The
// pages print no backward formulas; this is the chain rule through the
// forward pass, with the gate reading that the output depends on g_i only
// through the factor sigmoid(g_i) on selected rows.
//
// For a softmax row with probabilities P, output o and upstream gradient e:
//   dV += P^T e,  dP = e V^T,  D = <e, o>,  dS = P (dP - D),
//   dQ = scale dS K,  dK = scale dS^T Q.
// Local rows take e = dout; selected rows take e = sigmoid(g) dout on their
// global branch; dL/dg_i = sigmoid'(g_i) sum_h <dout_hi, global_hi>.
//
// Kernels, in launch order:
//   prep_dense   D for every local row: <dout, out> (CUDA cores, HBM-bound);
//                clears the row-to-selection map and the gate gradient.
//   prep_sel     per selected row: gathers Q and sigmoid(g) dout into compact
//                [Hq][cap][d] tensors, D of the global row, D of the local row
//                from the local branch the forward saved (the merged output
//                would bring back the rounding of sigmoid(g) global, which
//                does not cancel where dP and D should), the gate gradient and
//                the row-to-selection map.
//   dq (global)  one 128-row tile of compact selected rows per CTA: recompute
//                S = Q K^T and dP = dO V^T, dS into TMEM, dQ += dS K; fp32
//                result kept in the workspace.
//   dq (local)   the same over the window for every row; the epilogue adds the
//                global share of selected rows and writes bf16 dQ.
//   dkdv         one 128-key tile per CTA, K and V resident in shared memory;
//                loops over the query tiles that read it (window rows of every
//                head of the GQA group, then selected rows): S^T = K Q^T,
//                dP^T = V dO^T, P^T and dS^T into TMEM, dV += P^T dO,
//                dK += dS^T Q, both accumulated in TMEM.
//
// P uses the log-sum-exp the forward saved, so no online maximum is needed.
// TMEM bf16 tiles use a per-half layout: the half of the 128 columns a
// warpgroup owns is overwritten in place by its own 64 bf16 values (32
// columns), so the two warpgroups never wait for each other.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cstdint>
#include <type_traits>

#include "kernels.cuh"
#include "ptx.cuh"

namespace logo {

namespace {

constexpr int kBwdThreads = 64 + 256;  // TMA warp, MMA warp, two softmax warpgroups

__device__ __forceinline__ int ceil_div_i(int a, int b) { return (a + b - 1) / b; }

__device__ __forceinline__ uint8_t* align1024_b(uint8_t* p)
{
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// ------------------------------------------------------------------ prep

template <int D>
__global__ void __launch_bounds__(256) prep_dense_kernel(const PrepParams p)
{
    constexpr int kPer = D / 32;  // elements per lane
    const int lane = threadIdx.x & 31;
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    const long long rows = (long long)p.B * p.Hq * p.L;
    for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows; row += nwarps) {
        const uint16_t* e = p.dout + row * D + lane * kPer;
        const uint16_t* o = p.out + row * D + lane * kPer;
        float acc = 0.f;
        if (kPer == 4) {
            const uint2 ev = *reinterpret_cast<const uint2*>(e);
            const uint2 ov = *reinterpret_cast<const uint2*>(o);
            acc = bf16_lo(ev.x) * bf16_lo(ov.x) + bf16_hi(ev.x) * bf16_hi(ov.x) + bf16_lo(ev.y) * bf16_lo(ov.y) +
                  bf16_hi(ev.y) * bf16_hi(ov.y);
        } else {
            const uint32_t ev = *reinterpret_cast<const uint32_t*>(e);
            const uint32_t ov = *reinterpret_cast<const uint32_t*>(o);
            acc = bf16_lo(ev) * bf16_lo(ov) + bf16_hi(ev) * bf16_hi(ov);
        }
        #pragma unroll
        for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
        if (lane == 0) p.dl[row] = acc;
    }
    const long long grows = (long long)p.B * p.L;
    for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < grows;
         t += (long long)gridDim.x * blockDim.x) {
        p.slot[t] = -1;
        p.dgate[t] = 0.f;
    }
}

template <int D>
__global__ void __launch_bounds__(256) prep_sel_kernel(const PrepParams p)
{
    constexpr int kPer = D / 32;
    const int lane = threadIdx.x & 31;
    const int total = p.cu_sel[p.nseq];
    if (total > p.sel_stride || total < 0) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(p.status, kStatusBadArgument);
        return;
    }
    const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= p.sel_stride) return;
    if (r >= total) {
        // Rows past the selection: zero, so tiles that overhang the list read finite values.
        for (int h = 0; h < p.Hq; ++h) {
            const size_t base = ((size_t)h * p.sel_stride + r) * D + lane * kPer;
            #pragma unroll
            for (int u = 0; u < kPer; ++u) {
                p.q_sel[base + u] = 0;
                p.do_sel[base + u] = 0;
            }
        }
        return;
    }
    // The sequence whose list holds row r: cu_sel[s] <= r < cu_sel[s + 1].
    int lo = 0, hi = p.nseq;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.cu_sel[mid] <= r) lo = mid;
        else hi = mid;
    }
    const int s = lo;
    const long long b = p.cu_seqlens ? 0 : s;
    const long long s0 = p.cu_seqlens ? p.cu_seqlens[s] : 0;
    const long long t = s0 + p.sel_idx[r];
    const long long grow = b * p.L + t;
    const float sg = 1.f / (1.f + expf(-p.gate[grow]));
    float esum = 0.f;
    for (int h = 0; h < p.Hq; ++h) {
        const long long drow = ((b * p.Hq + h) * (long long)p.L + t) * D + lane * kPer;
        const size_t srow = ((size_t)h * p.sel_stride + r) * D + lane * kPer;
        float ev[kPer], ov[kPer], gv[kPer];
        #pragma unroll
        for (int u = 0; u < kPer; ++u) {
            ev[u] = __uint_as_float((uint32_t)p.dout[drow + u] << 16);
            ov[u] = __uint_as_float((uint32_t)p.loc_sel[srow + u] << 16);
            gv[u] = __uint_as_float((uint32_t)p.glob[srow + u] << 16);
            p.q_sel[srow + u] = p.q[drow + u];
        }
        float c = 0.f, o = 0.f, dg = 0.f;
        #pragma unroll
        for (int u = 0; u < kPer; ++u) {
            c += ev[u] * gv[u];
            o += ev[u] * ov[u];
            const __nv_bfloat16 es = __float2bfloat16_rn(sg * ev[u]);
            p.do_sel[srow + u] = __bfloat16_as_ushort(es);
            dg += __bfloat162float(es) * gv[u];
        }
        #pragma unroll
        for (int k = 16; k > 0; k >>= 1) {
            c += __shfl_xor_sync(0xffffffffu, c, k);
            o += __shfl_xor_sync(0xffffffffu, o, k);
            dg += __shfl_xor_sync(0xffffffffu, dg, k);
        }
        if (lane == 0) {
            p.ds_sel[(size_t)h * p.sel_stride + r] = dg;
            p.dl[(b * p.Hq + h) * (long long)p.L + t] = o;
        }
        esum += c;
    }
    if (lane == 0) {
        p.dgate[grow] = sg * (1.f - sg) * esum;
        p.slot[grow] = r;
    }
}

// ------------------------------------------------------------------ dQ

template <int D>
struct DqGeo {
    static constexpr int kChunkBytes = 128 * 128;
    static constexpr int kTile = 128 * D * 2;
    static constexpr int kKStages = 3;   // K(j) feeds S(j) and, two tiles later, dQ(j)
    static constexpr int kVStages = 2;
    static constexpr int kQOff = 0;
    static constexpr int kDoOff = kTile;
    static constexpr int kKOff = 2 * kTile;
    static constexpr int kVOff = kKOff + kKStages * kTile;
    static constexpr int kBarOff = kVOff + kVStages * kTile;
    static constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 2 + 1 + 1 + 1 + 1;
    static constexpr int kBytes = kBarOff + kNumBars * 8 + 16;
    static constexpr uint32_t kTmemS = 0;      // S(j) at column 128 * (j & 1)
    static constexpr uint32_t kTmemDP = 256;   // dP, overwritten in place by dS (bf16)
    static constexpr uint32_t kTmemDQ = 384;   // dQ accumulator, D columns
};

struct DqWork {
    int valid, b, s0, len, head, zq, row0, nrows, sel_base, min_pos, max_pos, kv_lo, n_kv;
};

template <int MODE>
__device__ DqWork dq_work(const BwdParams& p)
{
    DqWork w;
    w.valid = 0;
    const int seq = blockIdx.z;
    if (p.cu_seqlens) {
        w.b = 0;
        w.s0 = p.cu_seqlens[seq];
        w.len = p.cu_seqlens[seq + 1] - w.s0;
    } else {
        w.b = seq;
        w.s0 = 0;
        w.len = p.L;
    }
    if (w.len <= 0) return w;
    // Local rows: x = row tile, y = head.  Selected rows: x = head, y = chunk, heaviest chunk
    // first, so the longest prefixes of every head start in the first wave (chunk-fastest order
    // left the last head's longest prefixes for the tail: 2.37 against 2.21 ms at 32K).
    w.head = MODE == kModeLocal ? blockIdx.y : blockIdx.x;
    w.zq = w.b * p.Hq + w.head;
    if (MODE == kModeLocal) {
        w.row0 = blockIdx.x * 128;
        if (w.row0 >= w.len) return w;
        w.nrows = min(128, w.len - w.row0);
        w.min_pos = w.row0;
        w.max_pos = w.row0 + w.nrows - 1;
        w.kv_lo = max(0, w.min_pos - p.window + 1);
        w.sel_base = 0;
    } else {
        w.sel_base = p.cu_sel[seq];
        const int k = p.cu_sel[seq + 1] - w.sel_base;
        if (k > p.max_selected || p.cu_sel[seq + 1] > p.sel_stride) {
            if (threadIdx.x == 0) atomicOr(p.status, kStatusBadArgument);
            return w;
        }
        const int c = ceil_div_i(k, 128) - 1 - (int)blockIdx.y;  // heaviest chunk first
        if (c < 0) return w;
        w.row0 = c * 128;
        w.nrows = min(128, k - w.row0);
        w.min_pos = p.sel_idx[w.sel_base + w.row0];
        w.max_pos = p.sel_idx[w.sel_base + w.row0 + w.nrows - 1];
        w.kv_lo = 0;
    }
    w.n_kv = ceil_div_i(w.max_pos + 1 - w.kv_lo, 128);
    w.valid = 1;
    return w;
}

template <int D, int MODE>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_dq_kernel(const __grid_constant__ BwdParams p)
{
    using Geo = DqGeo<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024_b(smem_raw);
    uint8_t* sQ = smem + Geo::kQOff;
    uint8_t* sDo = smem + Geo::kDoOff;
    uint8_t* sK = smem + Geo::kKOff;
    uint8_t* sV = smem + Geo::kVOff;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Geo::kBarOff);
    uint64_t* qd_full = bars;
    uint64_t* k_full = qd_full + 1;
    uint64_t* k_empty = k_full + Geo::kKStages;
    uint64_t* v_full = k_empty + Geo::kKStages;
    uint64_t* v_empty = v_full + Geo::kVStages;
    uint64_t* s_full = v_empty + Geo::kVStages;  // [2]
    uint64_t* dp_full = s_full + 2;
    uint64_t* ds_full = dp_full + 1;             // 256 arrivals
    uint64_t* dq_full = ds_full + 1;
    uint64_t* drain = dq_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    __shared__ int sh_skip;
    if (threadIdx.x == 0) sh_skip = (*reinterpret_cast<volatile uint32_t*>(p.status) & kStatusTimeout) ? 1 : 0;
    __syncthreads();
    if (sh_skip) return;

    const DqWork w = dq_work<MODE>(p);
    if (!w.valid) return;

    if (threadIdx.x == 0) {
        mbar_init(qd_full, 1);
        for (int s = 0; s < Geo::kKStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < Geo::kVStages; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        mbar_init(&s_full[0], 1);
        mbar_init(&s_full[1], 1);
        mbar_init(dp_full, 1);
        mbar_init(ds_full, 256);
        mbar_init(dq_full, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t limit = p.timeout_ns;
    const int n_kv = w.n_kv;
    const int zkv = w.b * p.Hkv + w.head / p.G;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_kv = policy_evict_last();
            const uint64_t pol_q = policy_evict_first();
            const CUtensorMap* mq = MODE == kModeLocal ? &p.tm_q : &p.tm_qs;
            const CUtensorMap* mdo = MODE == kModeLocal ? &p.tm_do : &p.tm_dos;
            const int qrow = MODE == kModeLocal ? w.s0 + w.row0 : w.sel_base + w.row0;
            const int qslab = MODE == kModeLocal ? w.zq : w.head;
            mbar_arrive_expect_tx(qd_full, 2 * Geo::kTile);
            for (int c = 0; c < D / 64; ++c) {
                tma_load_3d(sQ + c * Geo::kChunkBytes, mq, qd_full, c * 64, qrow, qslab, pol_q);
                tma_load_3d(sDo + c * Geo::kChunkBytes, mdo, qd_full, c * 64, qrow, qslab, pol_q);
            }
            bool ok = true;
            int nk = 0, nv = 0;  // K and V tiles issued
            for (int j = 0; j < n_kv && ok; ++j) {
                const int row = w.s0 + w.kv_lo + j * 128;
                const int ks = j % Geo::kKStages;
                if (j >= Geo::kKStages)
                    ok = mbar_wait(&k_empty[ks], ((j / Geo::kKStages) - 1) & 1, abort_flag, p.status, limit);
                if (!ok) break;
                mbar_arrive_expect_tx(&k_full[ks], Geo::kTile);
                ++nk;
                for (int c = 0; c < D / 64; ++c)
                    tma_load_3d(sK + ks * Geo::kTile + c * Geo::kChunkBytes, &p.tm_k, &k_full[ks], c * 64, row, zkv,
                                pol_kv);
                const int vs = j % Geo::kVStages;
                if (j >= Geo::kVStages)
                    ok = mbar_wait(&v_empty[vs], ((j / Geo::kVStages) - 1) & 1, abort_flag, p.status, limit);
                if (!ok) break;
                mbar_arrive_expect_tx(&v_full[vs], Geo::kTile);
                ++nv;
                for (int c = 0; c < D / 64; ++c)
                    tma_load_3d(sV + vs * Geo::kTile + c * Geo::kChunkBytes, &p.tm_v, &v_full[vs], c * 64, row, zkv,
                                pol_kv);
            }
            if (*abort_flag) {
                volatile int dummy = 0;
                // stage s was armed (n - s + stages - 1) / stages times; wait for its last fill
                for (int s = 0; s < Geo::kKStages && s < nk; ++s)
                    mbar_wait(&k_full[s], ((nk - s + Geo::kKStages - 1) / Geo::kKStages - 1) & 1, &dummy, nullptr, limit);
                for (int s = 0; s < Geo::kVStages && s < nv; ++s)
                    mbar_wait(&v_full[s], ((nv - s + Geo::kVStages - 1) / Geo::kVStages - 1) & 1, &dummy, nullptr, limit);
                mbar_wait(qd_full, 0, &dummy, nullptr, limit);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ tcgen05 issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
            constexpr uint32_t idesc_dq = idesc_bf16_f32(128, D, true);
            const uint32_t sQa = smem_u32(sQ), sDoa = smem_u32(sDo), sKa = smem_u32(sK), sVa = smem_u32(sV);
            // D[128 x 128] = A[128 x D] B[128 x D]^T, both K-major tiles.
            // Each operand's descriptor is made once per call; the slice at byte offset `off`
            // is that descriptor plus off >> 4 (the start-address field is the low 14 bits and
            // every shared-memory address here is below 2^18, so the sum never carries out).
            auto issue_kmajor = [&](uint32_t d_tmem, uint32_t a_base, uint32_t b_base) {
                const uint64_t a0 = sdesc_sw128(a_base, 16, 1024), b0 = sdesc_sw128(b_base, 16, 1024);
                #pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = (uint64_t)((kk >> 2) * (Geo::kChunkBytes >> 4) + (kk & 3) * 2);
                    umma_ss(d_tmem, a0 + off, b0 + off, idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            // dQ += dS K: dS from TMEM (keys 0-63 in columns 0-31, keys 64-127 in 64-95).
            auto issue_dq = [&](int ks, bool first) {
                const uint64_t b0 = sdesc_sw128(sKa + ks * Geo::kTile, Geo::kChunkBytes, 1024);
                #pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a = tmem + Geo::kTmemDP + (kk >> 2) * 64 + (kk & 3) * 8;
                    const uint64_t b = b0 + (uint64_t)(kk * (2048 >> 4));
                    umma_ts(tmem + Geo::kTmemDQ, a, b, idesc_dq, (!first || kk > 0) ? 1u : 0u);
                }
            };
            bool ok = mbar_wait(qd_full, 0, abort_flag, p.status, limit);
            if (ok) ok = mbar_wait(&k_full[0], 0, abort_flag, p.status, limit);
            if (ok) {
                tc_fence_after();
                issue_kmajor(tmem + Geo::kTmemS, sQa, sKa);
                umma_commit(&s_full[0]);
                ok = mbar_wait(&v_full[0], 0, abort_flag, p.status, limit);
            }
            if (ok) {
                tc_fence_after();
                issue_kmajor(tmem + Geo::kTmemDP, sDoa, sVa);
                umma_commit(dp_full);
                umma_commit(&v_empty[0]);
                if (n_kv > 1) {
                    ok = mbar_wait(&k_full[1], 0, abort_flag, p.status, limit);
                    if (ok) {
                        tc_fence_after();
                        issue_kmajor(tmem + Geo::kTmemS + 128, sQa, sKa + Geo::kTile);
                        umma_commit(&s_full[1]);
                    }
                }
            }
            for (int j = 0; j < n_kv && ok; ++j) {
                ok = mbar_wait(ds_full, j & 1, abort_flag, p.status, limit);
                if (!ok) break;
                tc_fence_after();
                const int ks = j % Geo::kKStages;
                issue_dq(ks, j == 0);
                umma_commit(&k_empty[ks]);
                if (j + 1 < n_kv) {
                    const int vs = (j + 1) % Geo::kVStages;
                    ok = mbar_wait(&v_full[vs], ((j + 1) / Geo::kVStages) & 1, abort_flag, p.status, limit);
                    if (!ok) break;
                    tc_fence_after();
                    issue_kmajor(tmem + Geo::kTmemDP, sDoa, sVa + vs * Geo::kTile);
                    umma_commit(dp_full);
                    umma_commit(&v_empty[vs]);
                }
                if (j + 2 < n_kv) {
                    const int ks2 = (j + 2) % Geo::kKStages;
                    ok = mbar_wait(&k_full[ks2], ((j + 2) / Geo::kKStages) & 1, abort_flag, p.status, limit);
                    if (!ok) break;
                    tc_fence_after();
                    issue_kmajor(tmem + Geo::kTmemS + 128 * (j & 1), sQa, sKa + ks2 * Geo::kTile);
                    umma_commit(&s_full[j & 1]);
                }
            }
            if (ok) umma_commit(dq_full);
            umma_commit(drain);
            volatile int dummy = 0;
            mbar_wait(drain, 0, &dummy, nullptr, limit);
        }
    } else {
        // ------------------------------------------------------------ softmax warpgroups
        const int half = (warp - 2) >> 2;  // key columns 64*half .. 64*half+63
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;  // query row = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const bool row_valid = r < w.nrows;
        int pos;
        float lse2, dsum;
        if (MODE == kModeLocal) {
            pos = row_valid ? w.row0 + r : w.max_pos;
            const size_t idx = (size_t)w.zq * p.L + w.s0 + pos;
            lse2 = row_valid ? p.lse[idx] : INFINITY;
            dsum = row_valid ? p.dl[idx] : 0.f;
        } else {
            const size_t idx = (size_t)w.head * p.sel_stride + w.sel_base + w.row0 + r;
            pos = row_valid ? p.sel_idx[w.sel_base + w.row0 + r] : w.max_pos;
            lse2 = row_valid ? p.lse_s[idx] : INFINITY;
            dsum = row_valid ? p.ds_sel[idx] : 0.f;
        }
        const float sl2 = p.scale_log2;
        const int W = p.window;
        bool ok = true;
        for (int j = 0; j < n_kv; ++j) {
            const int buf = j & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[buf], (j >> 1) & 1, abort_flag, p.status, limit));
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[2][32];
            const uint32_t tS = tmem + lane_off + Geo::kTmemS + 128 * buf + 64 * half;
            tmem_ld32(tS, sr[0]);
            tmem_ld32(tS + 32, sr[1]);
            tmem_wait_ld(sr[0]);
            tmem_wait_ld(sr[1]);
            const int kbase = w.kv_lo + j * 128 + 64 * half;
            const bool need_mask = (kbase + 63 > w.min_pos) || (MODE == kModeLocal && kbase < w.max_pos - W + 1);
            const int hi = pos - kbase;
            const int lo = (MODE == kModeLocal) ? pos - W + 1 - kbase : INT_MIN;
            // P = exp2(S * scale * log2(e) - lse); the mask as selects behind a uniform test.
            // Paired fp32 instructions: x = S * sl2 - lse for two columns at once.
            const uint64_t sl2x2 = f2_pack(sl2, sl2), nlse2 = f2_pack(-lse2, -lse2);
            if (need_mask) {
                #pragma unroll
                for (int c = 0; c < 2; ++c) {
                    #pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const int col = c * 32 + e;
                        float x0, x1;
                        f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1])), sl2x2, nlse2),
                                  x0, x1);
                        sr[c][e] = __float_as_uint(fast_exp2((col <= hi) & (col >= lo) ? x0 : -INFINITY));
                        sr[c][e + 1] = __float_as_uint(fast_exp2((col + 1 <= hi) & (col + 1 >= lo) ? x1 : -INFINITY));
                    }
                }
            } else {
                #pragma unroll
                for (int c = 0; c < 2; ++c) {
                    #pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        float x0, x1;
                        f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1])), sl2x2, nlse2),
                                  x0, x1);
                        sr[c][e] = __float_as_uint(fast_exp2(x0));
                        sr[c][e + 1] = __float_as_uint(fast_exp2(x1));
                    }
                }
            }
            ok = __all_sync(0xffffffffu, mbar_wait(dp_full, j & 1, abort_flag, p.status, limit));
            if (!ok) break;
            tc_fence_after();
            const uint32_t tD = tmem + lane_off + Geo::kTmemDP + 64 * half;
            #pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t dp[32];
                tmem_ld32(tD + 32 * c, dp);
                tmem_wait_ld(dp);
                uint32_t pk[16];
                const uint64_t ndsum2 = f2_pack(-dsum, -dsum);
                #pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    // dS = P * (dP - D), two columns per instruction
                    const uint64_t p2 = f2_pack(__uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1]));
                    const uint64_t dp2 = f2_pack(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1]));
                    float d0, d1;
                    f2_unpack(f2_mul(p2, f2_add(dp2, ndsum2)), d0, d1);
                    pk[e / 2] = pack_bf16x2(d0, d1);
                }
                // Columns 16c .. 16c+15 of this half: dP there has been read (chunk 0 above).
                tmem_st16(tD + 16 * c, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(ds_full);
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(dq_full, 0, abort_flag, p.status, limit));
        if (ok) {
            tc_fence_after();
            const uint32_t tQ = tmem + lane_off + Geo::kTmemDQ + (D / 2) * half;
            int slot = -1;
            if (MODE == kModeLocal && row_valid && p.dq_sel) slot = p.slot[(size_t)w.b * p.L + w.s0 + pos];
            #pragma unroll 1
            for (int c = 0; c < D / 64; ++c) {
                uint32_t acc[32];
                __syncwarp();
                tmem_ld32(tQ + 32 * c, acc);
                tmem_wait_ld(acc);
                if (!row_valid) continue;
                float vals[32];
                #pragma unroll
                for (int e = 0; e < 32; ++e) vals[e] = __uint_as_float(acc[e]) * p.scale;
                const int col0 = (D / 2) * half + 32 * c;
                if (MODE == kModeGlobal) {
                    float4* dst = reinterpret_cast<float4*>(
                        p.dq_sel + ((size_t)w.head * p.sel_stride + w.sel_base + w.row0 + r) * D + col0);
                    #pragma unroll
                    for (int u = 0; u < 8; ++u)
                        dst[u] = make_float4(vals[4 * u], vals[4 * u + 1], vals[4 * u + 2], vals[4 * u + 3]);
                } else {
                    if (slot >= 0) {
                        const float4* add =
                            reinterpret_cast<const float4*>(p.dq_sel + ((size_t)w.head * p.sel_stride + slot) * D + col0);
                        #pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const float4 a = add[u];
                            vals[4 * u] += a.x;
                            vals[4 * u + 1] += a.y;
                            vals[4 * u + 2] += a.z;
                            vals[4 * u + 3] += a.w;
                        }
                    }
                    int4* dst = reinterpret_cast<int4*>(p.dq + ((size_t)w.zq * p.L + w.s0 + pos) * D + col0);
                    #pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        int4 o;
                        o.x = (int)pack_bf16x2(vals[u * 8 + 0], vals[u * 8 + 1]);
                        o.y = (int)pack_bf16x2(vals[u * 8 + 2], vals[u * 8 + 3]);
                        o.z = (int)pack_bf16x2(vals[u * 8 + 4], vals[u * 8 + 5]);
                        o.w = (int)pack_bf16x2(vals[u * 8 + 6], vals[u * 8 + 7]);
                        dst[u] = o;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ dK, dV

constexpr int kKvThreads = kBwdThreads + 32;  // + one warp that stages the per-column data
constexpr int kColStages = 4;                  // column data runs up to four query tiles ahead

template <int D>
struct KvGeo {
    static constexpr int kChunkBytes = 128 * 128;
    static constexpr int kTile = 128 * D * 2;
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kTile;
    static constexpr int kQOff = 2 * kTile;             // [2] query tiles
    static constexpr int kDoOff = kQOff + 2 * kTile;    // [2] dout tiles
    static constexpr int kColOff = kDoOff + 2 * kTile;  // [kColStages][3][128]: position, lse, D per column
    static constexpr int kBarOff = kColOff + kColStages * 3 * 128 * 4;
    static constexpr int kNumBars = 1 + 2 * 4 + 2 * kColStages + 6;
    static constexpr int kBytes = kBarOff + kNumBars * 8 + 16 + 16;
    static constexpr uint32_t kTmemS = 0;    // S^T, overwritten in place by P^T (bf16)
    static constexpr uint32_t kTmemDP = 128; // dP^T, overwritten in place by dS^T
    static constexpr uint32_t kTmemDV = 256;
    static constexpr uint32_t kTmemDK = 256 + D;
};

// Warp roles: 0 TMA (K, V once; Q and dout tiles), 1 tcgen05 issuer, 2-9 softmax (two
// warpgroups, one per half of the 128 query columns), 10 per-column data (query position,
// log-sum-exp, D) into a ring of kColStages slots, so those loads never gate the copies.
template <int D>
__global__ void __launch_bounds__(kKvThreads) bwd_dkdv_kernel(const __grid_constant__ BwdParams p)
{
    using Geo = KvGeo<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024_b(smem_raw);
    uint8_t* sK = smem + Geo::kKOff;
    uint8_t* sV = smem + Geo::kVOff;
    uint8_t* sQ = smem + Geo::kQOff;
    uint8_t* sDo = smem + Geo::kDoOff;
    int* scol = reinterpret_cast<int*>(smem + Geo::kColOff);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Geo::kBarOff);
    uint64_t* kv_full = bars;
    uint64_t* q_full = kv_full + 1;     // [2]
    uint64_t* q_empty = q_full + 2;     // [2]: after dK of the tile
    uint64_t* do_full = q_empty + 2;    // [2]
    uint64_t* do_empty = do_full + 2;   // [2]: after dV of the tile
    uint64_t* col_full = do_empty + 2;  // [kColStages], 32 arrivals
    uint64_t* col_empty = col_full + kColStages;  // [kColStages], 256 arrivals
    uint64_t* s_full = col_empty + kColStages;
    uint64_t* dp_full = s_full + 1;
    uint64_t* s_read = dp_full + 1;    // 256 arrivals: S^T of the tile is in registers, its columns are free
    uint64_t* pd_full = s_read + 1;    // 256 arrivals: P^T and dS^T written over dP^T
    uint64_t* acc_full = pd_full + 1;
    uint64_t* drain = acc_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* sh_info = reinterpret_cast<int*>(tmem_slot + 2);  // r_start of the selected rows

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    __shared__ int sh_skip;
    if (threadIdx.x == 0) sh_skip = (*reinterpret_cast<volatile uint32_t*>(p.status) & kStatusTimeout) ? 1 : 0;
    __syncthreads();
    if (sh_skip) return;

    // ---- the CTA's key tile and the query tiles that read it (uniform across the CTA)
    const int seq = blockIdx.z;
    const int hk = blockIdx.y;
    int b, s0, len;
    if (p.cu_seqlens) {
        b = 0;
        s0 = p.cu_seqlens[seq];
        len = p.cu_seqlens[seq + 1] - s0;
    } else {
        b = seq;
        s0 = 0;
        len = p.L;
    }
    const int j0 = blockIdx.x * 128;
    if (len <= 0 || j0 >= len) return;
    int sel_base = 0, k_sel = 0;
    if (p.cu_sel) {
        sel_base = p.cu_sel[seq];
        k_sel = p.cu_sel[seq + 1] - sel_base;
        if (k_sel > p.max_selected || p.cu_sel[seq + 1] > p.sel_stride) {
            if (threadIdx.x == 0) atomicOr(p.status, kStatusBadArgument);
            return;
        }
    }
    if (threadIdx.x == 0) {
        // first selected row at or after j0 (the list is ascending)
        int lo = 0, hi = k_sel;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (p.sel_idx[sel_base + mid] < j0) lo = mid + 1;
            else hi = mid;
        }
        sh_info[0] = lo;
    }
    __syncthreads();
    const int r_start = sh_info[0];
    const int nl = ceil_div_i(min(len, j0 + 127 + p.window) - j0, 128);  // window rows
    const int ng = ceil_div_i(k_sel - r_start, 128);                      // selected rows
    const int per_head = nl + ng;
    const int nb = p.G * per_head;
    const int zkv = b * p.Hkv + hk;

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
            mbar_init(&do_full[s], 1);
            mbar_init(&do_empty[s], 1);
        }
        for (int s = 0; s < kColStages; ++s) {
            mbar_init(&col_full[s], 32);
            mbar_init(&col_empty[s], 256);
        }
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(s_read, 256);
        mbar_init(pd_full, 256);
        mbar_init(acc_full, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t limit = p.timeout_ns;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA: K, V once; Q and dout per tile
        if (lane == 0) {
            const uint64_t pol_kv = policy_evict_first();
            const uint64_t pol_q = policy_evict_last();
            mbar_arrive_expect_tx(kv_full, 2 * Geo::kTile);
            for (int c = 0; c < D / 64; ++c) {
                tma_load_3d(sK + c * Geo::kChunkBytes, &p.tm_k, kv_full, c * 64, s0 + j0, zkv, pol_kv);
                tma_load_3d(sV + c * Geo::kChunkBytes, &p.tm_v, kv_full, c * 64, s0 + j0, zkv, pol_kv);
            }
            bool ok = true;
            int nq = 0, ndo = 0;  // tiles whose copies were started
            for (int n = 0; n < nb && ok; ++n) {
                const int st = n & 1;
                const int h = hk * p.G + n / per_head;
                const int m = n % per_head;
                const bool local = m < nl;
                const int q0 = local ? j0 + 128 * m : r_start + 128 * (m - nl);
                const int row = local ? s0 + q0 : sel_base + q0;
                const int slab = local ? b * p.Hq + h : h;
                // dout of tile n - 2 is released after its dV, before its Q (after dK): copy dout first.
                if (n >= 2) ok = mbar_wait(&do_empty[st], ((n >> 1) - 1) & 1, abort_flag, p.status, limit);
                if (!ok) break;
                mbar_arrive_expect_tx(&do_full[st], Geo::kTile);
                ++ndo;
                for (int c = 0; c < D / 64; ++c)
                    tma_load_3d(sDo + st * Geo::kTile + c * Geo::kChunkBytes, local ? &p.tm_do : &p.tm_dos,
                                &do_full[st], c * 64, row, slab, pol_q);
                if (n >= 2) ok = mbar_wait(&q_empty[st], ((n >> 1) - 1) & 1, abort_flag, p.status, limit);
                if (!ok) break;
                mbar_arrive_expect_tx(&q_full[st], Geo::kTile);
                ++nq;
                for (int c = 0; c < D / 64; ++c)
                    tma_load_3d(sQ + st * Geo::kTile + c * Geo::kChunkBytes, local ? &p.tm_q : &p.tm_qs,
                                &q_full[st], c * 64, row, slab, pol_q);
            }
            volatile int dummy = 0;
            if (*abort_flag) {
                // stage s was filled (count - s + 1) / 2 times; wait for its last fill
                for (int s = 0; s < 2 && s < nq; ++s)
                    mbar_wait(&q_full[s], ((nq - s + 1) / 2 - 1) & 1, &dummy, nullptr, limit);
                for (int s = 0; s < 2 && s < ndo; ++s)
                    mbar_wait(&do_full[s], ((ndo - s + 1) / 2 - 1) & 1, &dummy, nullptr, limit);
            }
            // K and V always land before the CTA ends (the MMA thread may have given up first).
            mbar_wait(kv_full, 0, &dummy, nullptr, limit);
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------ per-column data ring
        bool ok = true;
        for (int n = 0; n < nb && ok; ++n) {
            const int cs = n % kColStages;
            if (n >= kColStages)
                ok = __all_sync(0xffffffffu, mbar_wait(&col_empty[cs], ((n / kColStages) - 1) & 1, abort_flag,
                                                       p.status, limit));
            if (!ok) break;
            const int h = hk * p.G + n / per_head;
            const int m = n % per_head;
            const bool local = m < nl;
            const int q0 = local ? j0 + 128 * m : r_start + 128 * (m - nl);
            int qp[4];
            float l2[4], dd[4];
            #pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = lane * 4 + u;
                qp[u] = 0;
                l2[u] = -INFINITY;  // minus the query's lse (a column past the end gets P = 0)
                dd[u] = 0.f;
                if (local) {
                    qp[u] = q0 + c;
                    if (qp[u] < len) {
                        const size_t idx = ((size_t)(b * p.Hq + h)) * p.L + s0 + qp[u];
                        l2[u] = -__ldg(p.lse + idx);
                        dd[u] = __ldg(p.dl + idx);
                    }
                } else if (q0 + c < k_sel) {
                    qp[u] = __ldg(p.sel_idx + sel_base + q0 + c);
                    const size_t idx = (size_t)h * p.sel_stride + sel_base + q0 + c;
                    l2[u] = -__ldg(p.lse_s + idx);
                    dd[u] = __ldg(p.ds_sel + idx);
                }
            }
            int* cpos = scol + cs * 384;
            *reinterpret_cast<int4*>(cpos + lane * 4) = make_int4(qp[0], qp[1], qp[2], qp[3]);
            *reinterpret_cast<float4*>(cpos + 128 + lane * 4) = make_float4(l2[0], l2[1], l2[2], l2[3]);
            *reinterpret_cast<float4*>(cpos + 256 + lane * 4) = make_float4(dd[0], dd[1], dd[2], dd[3]);
            mbar_arrive(&col_full[cs]);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ tcgen05 issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
            constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, true);
            const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV), sQa = smem_u32(sQ), sDoa = smem_u32(sDo);
            // Each operand's descriptor is made once per call; the slice at byte offset `off`
            // is that descriptor plus off >> 4 (the start-address field is the low 14 bits and
            // every shared-memory address here is below 2^18, so the sum never carries out).
            auto issue_kmajor = [&](uint32_t d_tmem, uint32_t a_base, uint32_t b_base) {
                const uint64_t a0 = sdesc_sw128(a_base, 16, 1024), b0 = sdesc_sw128(b_base, 16, 1024);
                #pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = (uint64_t)((kk >> 2) * (Geo::kChunkBytes >> 4) + (kk & 3) * 2);
                    umma_ss(d_tmem, a0 + off, b0 + off, idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            // acc += X^T-tile (bf16 in the dP^T columns) times a [128 x D] tile.  Queries 32c .. 32c+31
            // of warpgroup h sit in columns 64h + 32c + which * 16 .. +15 (which 0: P^T, 1: dS^T).
            auto issue_acc = [&](uint32_t d_tmem, int which, uint32_t b_base, bool first) {
                const uint64_t b0 = sdesc_sw128(b_base, Geo::kChunkBytes, 1024);
                #pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a = tmem + Geo::kTmemDP + (kk >> 2) * 64 + ((kk >> 1) & 1) * 32 + which * 16 +
                                       (kk & 1) * 8;
                    const uint64_t bd = b0 + (uint64_t)(kk * (2048 >> 4));
                    umma_ts(d_tmem, a, bd, idesc_acc, (!first || kk > 0) ? 1u : 0u);
                }
            };
            bool ok = mbar_wait(kv_full, 0, abort_flag, p.status, limit);
            if (ok) ok = mbar_wait(&q_full[0], 0, abort_flag, p.status, limit);
            if (ok) {
                tc_fence_after();
                issue_kmajor(tmem + Geo::kTmemS, sKa, sQa);
                umma_commit(s_full);
                ok = mbar_wait(&do_full[0], 0, abort_flag, p.status, limit);
            }
            if (ok) {
                tc_fence_after();
                issue_kmajor(tmem + Geo::kTmemDP, sVa, sDoa);
                umma_commit(dp_full);
            }
            // Per tile n: S^T(n+1) as soon as the softmax has read S^T(n); dV(n), dK(n) once P^T(n)
            // and dS^T(n) are in the dP^T columns; then dP^T(n+1) over them (tcgen05 MMAs from one
            // thread execute in issue order, so it writes only after dV(n) and dK(n) have read).
            for (int n = 0; n < nb && ok; ++n) {
                const int st = n & 1;
                const bool nxt = n + 1 < nb;
                if (nxt) {
                    ok = mbar_wait(s_read, n & 1, abort_flag, p.status, limit);
                    if (ok) ok = mbar_wait(&q_full[st ^ 1], ((n + 1) >> 1) & 1, abort_flag, p.status, limit);
                    if (!ok) break;
                    tc_fence_after();
                    issue_kmajor(tmem + Geo::kTmemS, sKa, sQa + (st ^ 1) * Geo::kTile);
                    umma_commit(s_full);
                }
                ok = mbar_wait(pd_full, n & 1, abort_flag, p.status, limit);
                if (!ok) break;
                tc_fence_after();
                issue_acc(tmem + Geo::kTmemDV, 0, sDoa + st * Geo::kTile, n == 0);
                umma_commit(&do_empty[st]);
                issue_acc(tmem + Geo::kTmemDK, 1, sQa + st * Geo::kTile, n == 0);
                umma_commit(&q_empty[st]);
                if (nxt) {
                    ok = mbar_wait(&do_full[st ^ 1], ((n + 1) >> 1) & 1, abort_flag, p.status, limit);
                    if (!ok) break;
                    tc_fence_after();
                    issue_kmajor(tmem + Geo::kTmemDP, sVa, sDoa + (st ^ 1) * Geo::kTile);
                    umma_commit(dp_full);
                }
            }
            if (ok) umma_commit(acc_full);
            umma_commit(drain);
            volatile int dummy = 0;
            mbar_wait(drain, 0, &dummy, nullptr, limit);
        }
    } else {
        // ------------------------------------------------------------ softmax warpgroups
        const int half = (warp - 2) >> 2;  // query columns 64*half .. 64*half+63
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;  // key row = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int kp = j0 + r;              // key position in the sequence
        const float sl2 = p.scale_log2;
        const int W = p.window;
        bool ok = true;
        for (int n = 0; n < nb; ++n) {
            const int cs = n % kColStages;
            const int m = n % per_head;
            const bool local = m < nl;
            const int* cpos = scol + cs * 384 + 64 * half;
            const float* cnlse = reinterpret_cast<const float*>(scol + cs * 384 + 128 + 64 * half);
            const float* cdd = reinterpret_cast<const float*>(scol + cs * 384 + 256 + 64 * half);
            ok = __all_sync(0xffffffffu, mbar_wait(&col_full[cs], (n / kColStages) & 1, abort_flag, p.status, limit));
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(s_full, n & 1, abort_flag, p.status, limit));
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[2][32];
            const uint32_t tS = tmem + lane_off + Geo::kTmemS + 64 * half;
            tmem_ld32(tS, sr[0]);
            tmem_ld32(tS + 32, sr[1]);
            tmem_wait_ld(sr[0]);
            tmem_wait_ld(sr[1]);
            // S^T is in registers: the next tile's S^T may go into these columns now.
            tc_fence_before();
            mbar_arrive(s_read);
            // Tile-wide test: every (key, query) pair of the tile inside the mask.
            const int q_first = cpos[0 - 64 * half];
            const int q_last = local ? q_first + 127 : INT_MAX;
            const bool need_mask = !(q_first >= j0 + 127 && (!local || q_last - j0 < W));
            const int wl = local ? W : INT_MAX;  // a query more than wl - 1 past the key is out
            // P^T = exp2(S^T * scale * log2(e) - lse(query)); the mask, where the tile needs it,
            // as selects (a per-element branch here costs more than the exponentials).
            const uint64_t sl2x2 = f2_pack(sl2, sl2);
            auto p_chunk = [&](int c, auto masked) {
                #pragma unroll
                for (int e4 = 0; e4 < 32; e4 += 4) {
                    const int col = c * 32 + e4;
                    const float4 nl4 = *reinterpret_cast<const float4*>(cnlse + col);  // -lse per column
                    int qa[4] = {0, 0, 0, 0};
                    if (decltype(masked)::value) {
                        const int4 q4 = *reinterpret_cast<const int4*>(cpos + col);
                        qa[0] = q4.x;
                        qa[1] = q4.y;
                        qa[2] = q4.z;
                        qa[3] = q4.w;
                    }
                    // x = S^T * sl2 - lse, two columns per paired instruction
                    float x[4];
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[c][e4]), __uint_as_float(sr[c][e4 + 1])), sl2x2,
                                     f2_pack(nl4.x, nl4.y)),
                              x[0], x[1]);
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[c][e4 + 2]), __uint_as_float(sr[c][e4 + 3])), sl2x2,
                                     f2_pack(nl4.z, nl4.w)),
                              x[2], x[3]);
                    #pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        if (decltype(masked)::value) {
                            const int dq = qa[t] - kp;
                            x[t] = (dq >= 0) & (dq < wl) ? x[t] : -INFINITY;
                        }
                        sr[c][e4 + t] = __float_as_uint(fast_exp2(x[t]));
                    }
                }
            };
            if (need_mask) {
                p_chunk(0, std::true_type{});
                p_chunk(1, std::true_type{});
            } else {
                p_chunk(0, std::false_type{});
                p_chunk(1, std::false_type{});
            }
            ok = __all_sync(0xffffffffu, mbar_wait(dp_full, n & 1, abort_flag, p.status, limit));
            if (!ok) break;
            tc_fence_after();
            const uint32_t tD = tmem + lane_off + Geo::kTmemDP + 64 * half;
            #pragma unroll
            for (int c = 0; c < 2; ++c) {
                // dP^T columns 32c .. 32c+31 of this warpgroup, then P^T and dS^T of the same
                // 32 queries over exactly those columns (16 each).
                uint32_t dp[32];
                tmem_ld32(tD + 32 * c, dp);
                tmem_wait_ld(dp);
                uint32_t pp[16], pk[16];
                #pragma unroll
                for (int e4 = 0; e4 < 32; e4 += 4) {
                    const float4 d4 = *reinterpret_cast<const float4*>(cdd + c * 32 + e4);
                    // dS^T = P^T * (dP^T - D), two columns per paired instruction
                    float ds[4];
                    f2_unpack(f2_mul(f2_pack(__uint_as_float(sr[c][e4]), __uint_as_float(sr[c][e4 + 1])),
                                     f2_sub(f2_pack(__uint_as_float(dp[e4]), __uint_as_float(dp[e4 + 1])),
                                            f2_pack(d4.x, d4.y))),
                              ds[0], ds[1]);
                    f2_unpack(f2_mul(f2_pack(__uint_as_float(sr[c][e4 + 2]), __uint_as_float(sr[c][e4 + 3])),
                                     f2_sub(f2_pack(__uint_as_float(dp[e4 + 2]), __uint_as_float(dp[e4 + 3])),
                                            f2_pack(d4.z, d4.w))),
                              ds[2], ds[3]);
                    pk[e4 / 2] = pack_bf16x2(ds[0], ds[1]);
                    pk[e4 / 2 + 1] = pack_bf16x2(ds[2], ds[3]);
                    pp[e4 / 2] = pack_bf16x2(__uint_as_float(sr[c][e4]), __uint_as_float(sr[c][e4 + 1]));
                    pp[e4 / 2 + 1] = pack_bf16x2(__uint_as_float(sr[c][e4 + 2]), __uint_as_float(sr[c][e4 + 3]));
                }
                tmem_st16(tD + 32 * c, pp);
                tmem_st16(tD + 32 * c + 16, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(pd_full);
            mbar_arrive(&col_empty[cs]);  // this tile's column data has been read
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, p.status, limit));
        if (ok) {
            tc_fence_after();
            const bool row_valid = kp < len;
            const size_t orow = ((size_t)zkv * p.L + s0 + kp) * D;
            #pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                const uint32_t tA = tmem + lane_off + (which ? Geo::kTmemDK : Geo::kTmemDV) + (D / 2) * half;
                const float mul = which ? p.scale : 1.f;
                uint16_t* dst_base = (which ? p.dk : p.dv) + orow + (D / 2) * half;
                #pragma unroll 1
                for (int c = 0; c < D / 64; ++c) {
                    uint32_t acc[32];
                    __syncwarp();
                    tmem_ld32(tA + 32 * c, acc);
                    tmem_wait_ld(acc);
                    if (!row_valid) continue;
                    int4* dst = reinterpret_cast<int4*>(dst_base + 32 * c);
                    #pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        int4 o;
                        o.x = (int)pack_bf16x2(__uint_as_float(acc[u * 8 + 0]) * mul, __uint_as_float(acc[u * 8 + 1]) * mul);
                        o.y = (int)pack_bf16x2(__uint_as_float(acc[u * 8 + 2]) * mul, __uint_as_float(acc[u * 8 + 3]) * mul);
                        o.z = (int)pack_bf16x2(__uint_as_float(acc[u * 8 + 4]) * mul, __uint_as_float(acc[u * 8 + 5]) * mul);
                        o.w = (int)pack_bf16x2(__uint_as_float(acc[u * 8 + 6]) * mul, __uint_as_float(acc[u * 8 + 7]) * mul);
                        dst[u] = o;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <typename K>
cudaError_t launch_big(K kern, size_t smem, dim3 grid, const BwdParams& p, cudaStream_t stream,
                       int threads = kBwdThreads)
{
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, threads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_prep(const PrepParams& p, int d, cudaStream_t stream)
{
    const long long rows = (long long)p.B * p.Hq * p.L;
    if (rows > 0) {
        const long long blocks = (rows + 7) / 8;
        const int grid = (int)(blocks < 148 * 16 ? blocks : 148 * 16);
        if (d == 64) prep_dense_kernel<64><<<grid, 256, 0, stream>>>(p);
        else prep_dense_kernel<128><<<grid, 256, 0, stream>>>(p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (p.sel_stride > 0 && p.cu_sel) {
        const int grid = (p.sel_stride + 7) / 8;
        if (d == 64) prep_sel_kernel<64><<<grid, 256, 0, stream>>>(p);
        else prep_sel_kernel<128><<<grid, 256, 0, stream>>>(p);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

cudaError_t launch_bwd_dq(int mode, int d, const BwdParams& p, int max_seqlen, cudaStream_t stream)
{
    dim3 grid;
    if (mode == kModeLocal) grid = dim3((max_seqlen + 127) / 128, p.Hq, p.nseq);
    else grid = dim3(p.Hq, (p.max_selected + 127) / 128, p.nseq);
    if (grid.x == 0 || grid.y == 0 || grid.z == 0) return cudaSuccess;
    if (d == 64) {
        const size_t smem = DqGeo<64>::kBytes + 1024;
        return mode == kModeLocal ? launch_big(bwd_dq_kernel<64, kModeLocal>, smem, grid, p, stream)
                                  : launch_big(bwd_dq_kernel<64, kModeGlobal>, smem, grid, p, stream);
    }
    const size_t smem = DqGeo<128>::kBytes + 1024;
    return mode == kModeLocal ? launch_big(bwd_dq_kernel<128, kModeLocal>, smem, grid, p, stream)
                              : launch_big(bwd_dq_kernel<128, kModeGlobal>, smem, grid, p, stream);
}

cudaError_t launch_bwd_dkdv(int d, const BwdParams& p, int max_seqlen, cudaStream_t stream)
{
    // x = key tile, y = key/value head: the CTAs that run together share one head's Q and dout
    // in L2 (head-fastest order balanced the tail no better and read 2.9x the DRAM bytes).
    const dim3 grid((max_seqlen + 127) / 128, p.Hkv, p.nseq);
    if (grid.x == 0 || grid.y == 0 || grid.z == 0) return cudaSuccess;
    if (d == 64) return launch_big(bwd_dkdv_kernel<64>, KvGeo<64>::kBytes + 1024, grid, p, stream, kKvThreads);
    return launch_big(bwd_dkdv_kernel<128>, KvGeo<128>::kBytes + 1024, grid, p, stream, kKvThreads);
}

size_t bwd_smem_bytes(int d)
{
    const size_t a = d == 64 ? DqGeo<64>::kBytes : DqGeo<128>::kBytes;
    const size_t b = d == 64 ? KvGeo<64>::kBytes : KvGeo<128>::kBytes;
    return (a > b ? a : b) + 1024;
}

}  // namespace logo
