// Local (sliding-window) and selected-query global attention forward
// kernels for sm_100a, with the gated merge fused into the global kernel's
// epilogue.
//
// Method sources (page titles and sections):
//  * "LoGo: Token-Level Dynamic Local-Global Attention", Abstract: a windowed
//    branch for every token, a whole-prefix branch only where a gate turns it
//    on, and kernels that skip the global work of the other queries.
//  * "Learning When to Attend", "The Architecture of Conditional Attention":
//    the global branch is exact softmax attention, evaluated only at the
//    chosen query positions.
//  * "Local-global attention", Variants (Gemma 2): causal; the windowed kind
//    ignores keys further back than the window.
//
// One CTA owns two 128-row query tiles that read the same key/value head:
// two heads of one GQA group on the same rows, or (group size odd) two
// consecutive row tiles of one head.  Each key/value tile is staged once in
// shared memory by TMA and feeds both query tiles.
//
// Warp roles (12 warps, three warpgroups):
//   warp 0       TMA producer: Q tiles (local mode) and the K/V slots.
//   warp 1       tcgen05 issuer (one thread): S_i = Q_i K^T into TMEM, then
//                O_i += P_i V with P_i read straight from TMEM.
//   warps 2-3    idle; with warps 0-1 they form the producer warpgroup, which
//                hands most of its registers to the softmax warpgroups
//                (setmaxnreg: 88 registers per thread there, 208 in the softmax).
//   warps 4-7    softmax for query tile 0: thread = row = TMEM lane, holding all
//                128 scores of its row, so the row maximum is a thread-local
//                reduction.
//   warps 8-11   the same for query tile 1.
// TMEM (512 columns): S_0 | S_1 | O_0 | O_1.  P_i (bf16 pairs) overwrites the
// first half of S_i once the row has been read into registers.
//
// Online softmax in fp32 with a lazily updated reference maximum: the
// accumulator is rescaled only when a row's maximum grows by more than 2^8
// (in exp2 units), which keeps P <= 256 and exact normalisation at the end.
//
// Issue order of the tensor pipe (per key tile j, per query tile i):
//   PV_i(j), S_i(j+1).  S_i(j+1) overwrites the TMEM columns of P_i(j) only
//   after PV_i(j) has read them, because tcgen05 MMAs from one thread execute
//   in issue order; and the commit that signals S_i(j+1) also covers
//   PV_i(j), so O_i may be rescaled as soon as S_i(j+1) is seen, and is, before
//   P_i(j) is published.
// The MMA-issuing thread is the pipe's bottleneck (it reaches every P barrier
// after the softmax has completed it), so it waits on as few barriers as the
// data flow allows: one per key/value pair (K(j+1) and V(j) travel together),
// one per published P.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"

namespace logo {


namespace {

// K/V staging: two slots of one K tile and one V tile each.  Slot j % 2 receives the
// pair (K(j+1), V(j)) in one transaction: PV(j) and S(j+1) are issued in the same
// step, so the two tiles are needed together.  K(0) goes alone into slot 1 first.
constexpr int kSlots = 2;
constexpr int kKStages = kSlots;
constexpr int kVStages = kSlots;
constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the max grows by > 2^8

template <int D>
struct Geometry {
    static constexpr int kChunks = D / 64;              // 128-byte column chunks of a row
    static constexpr int kChunkBytes = 128 * 128;       // one chunk of a 128-row tile
    static constexpr int kQBytes = kTileM * D * 2;
    static constexpr int kKVBytes = kTileN * D * 2;
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kQOff + kNumQ * kQBytes;
    static constexpr int kVOff = kKOff + kKStages * kKVBytes;
    static constexpr int kBarOff = kVOff + kVStages * kKVBytes;
    static constexpr int kNumBars = 1 + 2 * kSlots + 2 * kNumQ + 2;
    static constexpr int kBytes = kBarOff + kNumBars * 8 + 16;
    static constexpr int kTmemS = 0;          // S_i at column 128 * i
    static constexpr int kTmemO = 128 * kNumQ; // O_i at column 256 + D * i
    static constexpr uint32_t kTmemCols = 512;
};

// What one CTA computes; identical in every thread.
struct Work {
    int valid;
    int seq;            // sequence index
    int b;              // batch row of the slab (0 when packed)
    int s0;             // first row of the sequence in the slab
    int len;            // sequence length
    int hk;             // key/value head
    int head[kNumQ];    // query head of tile i
    int row0[kNumQ];    // local: first position; global: offset into the selection list
    int nrows[kNumQ];   // valid rows of tile i
    int sel_base;       // global: cu_sel[seq]
    int min_pos, max_pos;
    int kv_lo, n_kv;
};

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Debug build (-DLOGO_DEBUG_BOUNDS): every TMA coordinate, gathered row and stored
// row is checked against the tensor it addresses before the access.  A failed check
// sets kStatusBounds, raises the CTA's abort flag (so every wait of the CTA gives up at
// once) and the access is skipped.  In the normal build the checks compile away.
__device__ __forceinline__ bool in_bounds(bool ok, uint32_t* status, volatile int* abort_flag)
{
#ifdef LOGO_DEBUG_BOUNDS
    if (!ok) {
        atomicOr(status, kStatusBounds);
        *abort_flag = 1;
    }
    return ok;
#else
    (void)status;
    (void)abort_flag;
    return true;
#endif
}

template <int MODE>
__device__ Work make_work(const AttnParams& p)
{
    Work w;
    w.valid = 0;
    const int seq = blockIdx.z;
    w.seq = seq;
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
    if (MODE == kModeLocal) {
        if (p.pair_heads) {
            const int tile = gridDim.x - 1 - blockIdx.x;
            const int t0 = tile * kTileM;
            if (t0 >= w.len) return w;
            for (int i = 0; i < kNumQ; ++i) {
                w.head[i] = blockIdx.y * kNumQ + i;
                w.row0[i] = t0;
                w.nrows[i] = min(kTileM, w.len - t0);
            }
        } else {
            const int tile = gridDim.x - 1 - blockIdx.x;
            const int t0 = tile * kTileM * kNumQ;
            if (t0 >= w.len) return w;
            for (int i = 0; i < kNumQ; ++i) {
                w.head[i] = blockIdx.y;
                w.row0[i] = t0 + i * kTileM;
                w.nrows[i] = max(0, min(kTileM, w.len - w.row0[i]));
            }
        }
        w.min_pos = w.row0[0];
        w.max_pos = w.row0[0];
        for (int i = 0; i < kNumQ; ++i)
            if (w.nrows[i] > 0) w.max_pos = max(w.max_pos, w.row0[i] + w.nrows[i] - 1);
        w.kv_lo = max(0, w.min_pos - p.window + 1);
    } else {
        w.sel_base = p.cu_sel[seq];
        const int k = p.cu_sel[seq + 1] - w.sel_base;
        if (k > p.max_selected || k < 0 || w.sel_base < 0) {
            if (threadIdx.x == 0) atomicOr(p.status, kStatusBadArgument);
            return w;
        }
        if (k == 0) return w;
        if (p.lse && p.cu_sel[seq + 1] > p.sel_stride) {
            if (threadIdx.x == 0) atomicOr(p.status, kStatusBadArgument);
            return w;
        }
        const int nch = ceil_div(k, kTileM);
        if (p.pair_heads) {
            const int c = nch - 1 - (int)blockIdx.y;
            if (c < 0) return w;
            for (int i = 0; i < kNumQ; ++i) {
                w.head[i] = blockIdx.x * kNumQ + i;
                w.row0[i] = c * kTileM;
                w.nrows[i] = min(kTileM, k - c * kTileM);
            }
        } else {
            const int cp = ceil_div(nch, kNumQ) - 1 - (int)blockIdx.y;
            if (cp < 0) return w;
            for (int i = 0; i < kNumQ; ++i) {
                w.head[i] = blockIdx.x;
                w.row0[i] = (cp * kNumQ + i) * kTileM;
                w.nrows[i] = max(0, min(kTileM, k - w.row0[i]));
            }
        }
        const int32_t* sel = p.sel_idx + w.sel_base;
        w.min_pos = sel[w.row0[0]];
        w.max_pos = w.min_pos;
        for (int i = 0; i < kNumQ; ++i)
            if (w.nrows[i] > 0) w.max_pos = max(w.max_pos, sel[w.row0[i] + w.nrows[i] - 1]);
        // The list comes from the caller: a tile whose first or last position lies
        // outside the sequence is reported and skipped whole (its key range would be
        // meaningless).  Single rows out of order are caught where they are read.
        if (w.min_pos < 0 || w.max_pos >= w.len) {
            if (threadIdx.x == 0) atomicOr(p.status, kStatusBadArgument);
            return w;
        }
        w.kv_lo = 0;
    }
    w.hk = w.head[0] / p.G;
    w.n_kv = ceil_div(w.max_pos + 1 - w.kv_lo, kTileN);
    w.valid = 1;
    return w;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p)
{
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams p)
{
    using Geo = Geometry<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sQ = smem + Geo::kQOff;
    uint8_t* sK = smem + Geo::kKOff;
    uint8_t* sV = smem + Geo::kVOff;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Geo::kBarOff);
    uint64_t* q_full = bars;
    uint64_t* kv_full = q_full + 1;           // [kSlots]: the slot's tiles have landed
    uint64_t* kv_empty = kv_full + kSlots;    // [kSlots]: the MMAs that read the slot have completed
    uint64_t* s_full = kv_empty + kSlots;
    uint64_t* p_full = s_full + kNumQ;        // [kNumQ]: P_i written
    uint64_t* o_full = p_full + kNumQ;
    uint64_t* drain = o_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const Work w = make_work<MODE>(p);
    if (!w.valid) return;  // uniform across the CTA

    const int zkv = w.b * p.Hkv + w.hk;
    // Producer state: thread 0 (the TMA lane) starts the first copies (the Q tiles, K(0)) right
    // after it has initialised the barriers, before TMEM allocation and the CTA-wide sync.
    bool p_ok = true, q_armed = false;
    int armed[kSlots] = {0, 0};
    // A CTA launched after another one recorded a timeout does no work past its first copies,
    // so a broken launch ends quickly instead of waiting out every CTA's limit.  The status
    // word is read while those copies are issued.
    __shared__ int sh_skip;
    if (threadIdx.x == 0) {
        mbar_init(q_full, MODE == kModeLocal ? 1 : 128 * kNumQ);
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int i = 0; i < kNumQ; ++i) mbar_init(&s_full[i], 1);
        for (int i = 0; i < kNumQ; ++i) mbar_init(&p_full[i], 128);
        mbar_init(o_full, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        const uint32_t status0 = *reinterpret_cast<volatile uint32_t*>(p.status);
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_v);
        const int slabs = p.cu_seqlens ? 1 : p.nseq;  // batch rows of the tensors
        p_ok = in_bounds(zkv >= 0 && zkv < slabs * p.Hkv, p.status, abort_flag);
        // A tile with no rows (the second tile past a sequence's end) is still loaded:
        // its rows past the tensor's end read as zeros.
        for (int i = 0; i < kNumQ && p_ok && MODE == kModeLocal; ++i)
            p_ok = in_bounds(w.nrows[i] <= 0 || (w.s0 + w.row0[i] >= 0 && w.s0 + w.row0[i] < p.L &&
                                                 w.b * p.Hq + w.head[i] >= 0 && w.b * p.Hq + w.head[i] < slabs * p.Hq),
                             p.status, abort_flag);
        if (MODE == kModeLocal && p_ok) {
            q_armed = true;
            tma_prefetch_desc(&p.tm_q);
            const uint64_t pol_q = policy_evict_first();
            mbar_arrive_expect_tx(q_full, kNumQ * Geo::kQBytes);
            for (int i = 0; i < kNumQ; ++i)
                for (int c = 0; c < Geo::kChunks; ++c)
                    tma_load_3d(sQ + i * Geo::kQBytes + c * Geo::kChunkBytes, &p.tm_q, q_full, c * 64,
                                w.s0 + w.row0[i], w.b * p.Hq + w.head[i], pol_q);
        }
        // Transactions on slot s: use n of the slot (n = 0, 1, ...) completes phase n of
        // kv_full[s]; slot 1's use 0 is K(0) alone, then pair j sits in slot j % 2 as
        // that slot's use (j + (j & 1)) / 2.
        if (p_ok) p_ok = in_bounds(w.s0 + w.kv_lo >= 0 && w.s0 + w.kv_lo < p.L, p.status, abort_flag);
        if (p_ok) {
            mbar_arrive_expect_tx(&kv_full[1], Geo::kKVBytes);
            ++armed[1];
            for (int c = 0; c < Geo::kChunks; ++c)
                tma_load_3d(sK + 1 * Geo::kKVBytes + c * Geo::kChunkBytes, &p.tm_k, &kv_full[1], c * 64,
                            w.s0 + w.kv_lo, zkv, policy_evict_last());
        }
        sh_skip = (status0 & kStatusTimeout) ? 1 : 0;
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Geo::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t limit = p.timeout_ns;
    const int n_kv = w.n_kv;
    if (sh_skip) {
        if (threadIdx.x == 0) {
            // let the first copies land before the CTA exits
            volatile int dummy = 0;
            if (q_armed) mbar_wait(q_full, 0, &dummy, nullptr, limit);
            if (armed[1]) mbar_wait(&kv_full[1], 0, &dummy, nullptr, limit);
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 1) {
            tc_fence_after();
            tmem_dealloc(tmem, Geo::kTmemCols);
        }
        return;
    }

    if (warp < 4) {
      // Producer warpgroup: TMA (warp 0), tcgen05 issue (warp 1), two idle warps.
      // It hands registers to the softmax warpgroups.
      reg_dealloc<kProducerRegs>();
      if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            // Q and K(0) are in flight (started before the CTA-wide sync); the pairs follow.
            const uint64_t pol_kv = policy_evict_last();
            bool ok = p_ok;
            auto slot_use = [](int j) { return (j + (j & 1)) / 2; };
            for (int j = 0; j < n_kv && ok; ++j) {
                const int sl = j & 1;
                const int use = slot_use(j);
                const bool with_k = j + 1 < n_kv;
                const int row_v = w.s0 + w.kv_lo + j * kTileN;
                const int row_k = row_v + kTileN;
                if (!in_bounds(row_v >= 0 && row_v < p.L && (!with_k || row_k < p.L), p.status, abort_flag)) break;
                // the slot's previous contents have been read
                if (use >= 1) ok = mbar_wait(&kv_empty[sl], (use - 1) & 1, abort_flag, p.status, limit);
                if (!ok) break;
                mbar_arrive_expect_tx(&kv_full[sl], (with_k ? 2 : 1) * Geo::kKVBytes);
                ++armed[sl];
                for (int c = 0; c < Geo::kChunks; ++c)
                    tma_load_3d(sV + sl * Geo::kKVBytes + c * Geo::kChunkBytes, &p.tm_v, &kv_full[sl], c * 64, row_v,
                                zkv, pol_kv);
                if (with_k)
                    for (int c = 0; c < Geo::kChunks; ++c)
                        tma_load_3d(sK + sl * Geo::kKVBytes + c * Geo::kChunkBytes, &p.tm_k, &kv_full[sl], c * 64,
                                    row_k, zkv, pol_kv);
            }
            if (*abort_flag) {
                // Let every copy this thread started land before the CTA exits.
                volatile int dummy = 0;
                for (int s2 = 0; s2 < kSlots; ++s2)
                    if (armed[s2]) mbar_wait(&kv_full[s2], (armed[s2] - 1) & 1, &dummy, nullptr, limit);
                if (q_armed) mbar_wait(q_full, 0, &dummy, nullptr, limit);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ tcgen05 issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(kTileM, kTileN, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(kTileM, D, true);
            // Descriptors of each operand's first slice, made once; the slice at byte offset
            // `off` is the base plus off >> 4 (the start-address field is the low 14 bits and
            // every shared-memory address here is below 2^18, so the sum never carries out).
            const uint64_t dq0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t dk0 = sdesc_sw128(smem_u32(sK), 16, 1024);
            const uint64_t dv0 = sdesc_sw128(smem_u32(sV), Geo::kChunkBytes, 1024);
            auto issue_s = [&](int i, int ks) {
                const uint32_t d_tmem = tmem + Geo::kTmemS + 128 * i;
                const uint64_t a0 = dq0 + (uint64_t)(i * (Geo::kQBytes >> 4));
                const uint64_t b0 = dk0 + (uint64_t)(ks * (Geo::kKVBytes >> 4));
                #pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = (uint64_t)((kk >> 2) * (Geo::kChunkBytes >> 4) + (kk & 3) * 2);
                    umma_ss(d_tmem, a0 + off, b0 + off, idesc_qk, kk > 0 ? 1u : 0u);
                }
            };
            // O_i += P_i V over the 128 keys of the tile.
            auto issue_pv = [&](int i, int vs, bool first) {
                const uint32_t d_tmem = tmem + Geo::kTmemO + D * i;
                const uint32_t p_tmem = tmem + Geo::kTmemS + 128 * i;
                const uint64_t b0 = dv0 + (uint64_t)(vs * (Geo::kKVBytes >> 4));
                #pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_ts(d_tmem, p_tmem + kk * 8, b0 + (uint64_t)(kk * (2048 >> 4)), idesc_pv,
                            (!first || kk > 0) ? 1u : 0u);
            };
            bool ok = mbar_wait(q_full, 0, abort_flag, p.status, limit);
            if (ok) ok = mbar_wait(&kv_full[1], 0, abort_flag, p.status, limit);  // K(0)
            if (ok) {
                tc_fence_after();
                for (int i = 0; i < kNumQ; ++i) {
                    issue_s(i, 1);
                    umma_commit(&s_full[i]);
                }
                umma_commit(&kv_empty[1]);
            }
            for (int j = 0; j < n_kv && ok; ++j) {
                const bool nxt = j + 1 < n_kv;
                const int sl = j & 1;
                // V(j) and, if there is one, K(j+1): the slot's use (j + (j & 1)) / 2
                ok = mbar_wait(&kv_full[sl], ((j + (j & 1)) / 2) & 1, abort_flag, p.status, limit);
                if (!ok) break;
                tc_fence_after();
                for (int i = 0; i < kNumQ && ok; ++i) {
                    ok = mbar_wait(&p_full[i], j & 1, abort_flag, p.status, limit);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(i, sl, j == 0);
                    if (nxt) {
                        issue_s(i, sl);
                        umma_commit(&s_full[i]);
                    }
                }
                if (!ok) break;
                umma_commit(&kv_empty[sl]);
            }
            if (ok) umma_commit(o_full);
            // Drain: everything issued above completes before TMEM is released.
            umma_commit(drain);
            volatile int dummy = 0;
            mbar_wait(drain, 0, &dummy, nullptr, limit);
        }
      }
    } else {
        reg_alloc<kSoftmaxRegs>();
        // ------------------------------------------------------------ softmax warpgroups
        // One warpgroup per query tile; thread = row = TMEM lane, holding all 128
        // scores of its row, so the row maximum needs no exchange.
        const int wg = (warp - 4) >> 2;           // query tile
        const int quarter = warp & 3;             // TMEM lane quarter this warp may touch
        const int r = quarter * 32 + lane;        // row of the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_off + Geo::kTmemS + 128 * wg;  // S_wg, and P_wg over its first 64 columns
        const uint32_t tO = tmem + lane_off + Geo::kTmemO + D * wg;    // all D columns of O for this row
        // Per-tile fields picked with selects (no dynamic indexing into Work).
        const int my_nrows = wg ? w.nrows[1] : w.nrows[0];
        const int my_row0 = wg ? w.row0[1] : w.row0[0];
        bool row_valid = r < my_nrows;
        const int head = wg ? w.head[1] : w.head[0];
        const int zq = w.b * p.Hq + head;
        int pos;  // position of this row within its sequence
        if (MODE == kModeLocal) {
            pos = row_valid ? my_row0 + r : w.max_pos;
        } else {
            pos = w.max_pos;
            if (row_valid) {
                // Each entry must lie in [min_pos, max_pos] of its tile (so inside the
                // sequence and inside the tile's key range) and above the entry before
                // it; a row that breaks this is reported and neither read nor written.
                const int idx = my_row0 + r;
                const int32_t* sel = p.sel_idx + w.sel_base;
                const int x = sel[idx];
                const bool ok_row = x >= w.min_pos && x <= w.max_pos && (idx == 0 || x > sel[idx - 1]);
                if (ok_row) {
                    pos = x;
                } else {
                    row_valid = false;
                    atomicOr(p.status, kStatusBadArgument);
                }
            }
            row_valid = row_valid && in_bounds(zq >= 0 && zq < (p.cu_seqlens ? 1 : p.nseq) * p.Hq && pos >= 0 &&
                                                   pos < w.len && w.s0 + pos < p.L,
                                               p.status, abort_flag);
            // Gather this row of Q into the 128B-swizzled tile.
            uint8_t* dst = sQ + wg * Geo::kQBytes;
            const int4* src = reinterpret_cast<const int4*>(p.q + ((size_t)zq * p.L + w.s0 + pos) * D);
            constexpr int kUnits = Geo::kChunks * 8;  // 16-byte units per row
            #pragma unroll
            for (int u = 0; u < kUnits; ++u) {
                const int c = u >> 3, e = u & 7;
                const int4 val = row_valid ? __ldg(src + u) : make_int4(0, 0, 0, 0);
                *reinterpret_cast<int4*>(dst + c * Geo::kChunkBytes + r * 128 + ((e ^ (r & 7)) << 4)) = val;
            }
            fence_proxy_async_smem();
            mbar_arrive(q_full);
        }
        const float sl2 = p.scale_log2;
        const float resc_raw = kRescaleLog2 / sl2;  // threshold in raw score units
        float m_run = -INFINITY;  // reference max (raw units)
        uint64_t l2x = 0ull;      // row sum, two partial sums in one register pair
        bool ok = true;
        const int W = p.window;
        for (int j = 0; j < n_kv; ++j) {
            // Warp-uniform outcome: the tcgen05 loads below are warp-collective.
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[wg], j & 1, abort_flag, p.status, limit));
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[4][32];
            #pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, sr[c]);
            #pragma unroll
            for (int c = 0; c < 4; ++c) tmem_wait_ld(sr[c]);
            const int kbase = w.kv_lo + j * kTileN;  // position of the tile's first key
            const bool need_mask = (kbase + kTileN - 1 > w.min_pos) || (MODE == kModeLocal && kbase < w.max_pos - W + 1);
            if (need_mask) {
                const int hi = pos - kbase;                                          // keep column c <= hi
                const int lo = (MODE == kModeLocal) ? pos - W + 1 - kbase : INT_MIN;  // keep column c >= lo
                // Selects, not branches: a per-element branch costs more than the exponentials.
                #pragma unroll
                for (int c = 0; c < 4; ++c) {
                    #pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int col = c * 32 + e;
                        sr[c][e] = (col <= hi) & (col >= lo) ? sr[c][e] : __float_as_uint(-INFINITY);
                    }
                }
            }
            float mx[4];
            #pragma unroll
            for (int c = 0; c < 4; ++c) {
                mx[c] = fmaxf(__uint_as_float(sr[c][0]), __uint_as_float(sr[c][1]));
                #pragma unroll
                for (int e = 2; e < 32; e += 2) mx[c] = fmax3(mx[c], __uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1]));
            }
            const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            const float m_new = fmaxf(m_run, mt);
            const bool need = m_new > m_run + resc_raw;
            float alpha = 1.f;
            if (need) {
                alpha = (m_run == -INFINITY) ? 0.f : fast_exp2((m_run - m_new) * sl2);
                m_run = m_new;
                l2x = f2_mul(l2x, f2_pack(alpha, alpha));
            }
            const float mref = (m_run == -INFINITY) ? 0.f : m_run * sl2;
            // Paired fp32 instructions for the scaling and the row sums.
            const uint64_t sl2x2 = f2_pack(sl2, sl2), nmref2 = f2_pack(-mref, -mref);
            #pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pk[16];
                #pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float x0, x1, p0, p1;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1])), sl2x2, nmref2),
                              x0, x1);
                    p0 = fast_exp2(x0);
                    p1 = fast_exp2(x1);
                    l2x = f2_add(l2x, f2_pack(p0, p1));
                    pk[e / 2] = pack_bf16x2(p0, p1);
                }
                tmem_st16(tS + c * 16, pk);
                if (c == 3) {
                    // Rare: the row maximum grew past the threshold, so O must be rescaled
                    // before any PV of this tile (PV of tile j-1 is complete: the commit
                    // that signalled S(j) covers it).  The PV MMAs of the first P part
                    // write every column of O, so this comes before that part is published.
                    const bool any = __any_sync(0xffffffffu, need);  // also reconverges the warp
                    if (any && j > 0) {
                        #pragma unroll 1
                        for (int cc = 0; cc < D / 32; ++cc) {
                            uint32_t orr[32];
                            tmem_ld32(tO + cc * 32, orr);
                            tmem_wait_ld(orr);
                            #pragma unroll
                            for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
                            tmem_st32(tO + cc * 32, orr);
                        }
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&p_full[wg]);
                }
            }
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_full, 0, abort_flag, p.status, limit));
        if (ok) {
            tc_fence_after();
            float l_lo, l_hi;
            f2_unpack(l2x, l_lo, l_hi);
            const float l_row = l_lo + l_hi;
            const float inv_l = l_row > 0.f ? 1.f / l_row : 0.f;
            uint16_t* orow = p.out + ((size_t)zq * p.L + w.s0 + pos) * D;
            if (row_valid)
                row_valid = in_bounds(zq >= 0 && zq < (p.cu_seqlens ? 1 : p.nseq) * p.Hq && pos >= 0 && pos < w.len &&
                                          w.s0 + pos < p.L,
                                      p.status, abort_flag);
            // Saved for the backward pass: the row's log-sum-exp (exp2 domain) and,
            // for selected rows, the global branch before the gate.
            const size_t srow = MODE == kModeGlobal ? (size_t)head * p.sel_stride + w.sel_base + my_row0 + r : 0;
            if (p.lse && row_valid) {
                const float lse2 = l_row > 0.f ? m_run * sl2 + log2f(l_row) : INFINITY;
                if (MODE == kModeLocal) p.lse[(size_t)zq * p.L + w.s0 + pos] = lse2;
                else p.lse[srow] = lse2;
            }
            uint16_t* grow = (MODE == kModeGlobal && p.glob) ? p.glob + srow * D : nullptr;
            uint16_t* lrow = (MODE == kModeGlobal && p.loc_sel) ? p.loc_sel + srow * D : nullptr;
            float gsig = 0.f;
            if (MODE == kModeGlobal && p.merge && row_valid) {
                const float g = p.gate[(size_t)w.b * p.L + w.s0 + pos];
                gsig = 1.f / (1.f + expf(-g));
            }
            // All of O_i's columns in one round trip to TMEM, then normalise and store.
            uint32_t oall[D / 32][32];
            __syncwarp();
            #pragma unroll
            for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + c * 32, oall[c]);
            #pragma unroll
            for (int c = 0; c < D / 32; ++c) tmem_wait_ld(oall[c]);
            #pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                if (!row_valid) break;
                float vals[32];
                #pragma unroll
                for (int e = 0; e < 32; ++e) vals[e] = __uint_as_float(oall[c][e]) * inv_l;
                int4* dst = reinterpret_cast<int4*>(orow + c * 32);
                if (MODE == kModeGlobal && grow) {
                    int4* gdst = reinterpret_cast<int4*>(grow + c * 32);
                    #pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        int4 o;
                        o.x = (int)pack_bf16x2(vals[u * 8 + 0], vals[u * 8 + 1]);
                        o.y = (int)pack_bf16x2(vals[u * 8 + 2], vals[u * 8 + 3]);
                        o.z = (int)pack_bf16x2(vals[u * 8 + 4], vals[u * 8 + 5]);
                        o.w = (int)pack_bf16x2(vals[u * 8 + 6], vals[u * 8 + 7]);
                        gdst[u] = o;
                    }
                }
                if (MODE == kModeGlobal && p.merge) {
                    #pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        int4 loc = dst[u];
                        if (lrow) reinterpret_cast<int4*>(lrow + c * 32)[u] = loc;
                        const uint32_t lw[4] = {(uint32_t)loc.x, (uint32_t)loc.y, (uint32_t)loc.z, (uint32_t)loc.w};
                        #pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            const float lo = __uint_as_float(lw[t] << 16);
                            const float hi = __uint_as_float(lw[t] & 0xffff0000u);
                            vals[u * 8 + 2 * t] = fmaf(gsig, vals[u * 8 + 2 * t], lo);
                            vals[u * 8 + 2 * t + 1] = fmaf(gsig, vals[u * 8 + 2 * t + 1], hi);
                        }
                    }
                }
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

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Geo::kTmemCols);
    }
}

template <int D, int MODE>
cudaError_t launch_one(const AttnParams& p, dim3 grid, cudaStream_t stream)
{
    const size_t smem = Geometry<D>::kBytes + 1024;
    auto kern = attn_fwd_kernel<D, MODE>;
    // The register split (setmaxnreg) hands out exactly what the launch holds; a build
    // whose kernel was given fewer registers per thread would make the increase wait
    // forever, so it is refused here instead of launched.
    static const cudaError_t regs_ok = [&] {
        cudaFuncAttributes fa;
        cudaError_t r = cudaFuncGetAttributes(&fa, kern);
        if (r != cudaSuccess) return r;
        return (long)fa.numRegs * kThreads >= 128L * kProducerRegs + 128L * kNumQ * kSoftmaxRegs
                   ? cudaSuccess
                   : cudaErrorInvalidConfiguration;
    }();
    if (regs_ok != cudaSuccess) return regs_ok;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

size_t attn_smem_bytes(int d)
{
    return d == 64 ? Geometry<64>::kBytes + 1024 : Geometry<128>::kBytes + 1024;
}

cudaError_t launch_attn(int mode, int d, const AttnParams& p, int max_seqlen, cudaStream_t stream)
{
    dim3 grid;
    if (mode == kModeLocal) {
        const int tiles = p.pair_heads ? (max_seqlen + kTileM - 1) / kTileM
                                       : (max_seqlen + kTileM * kNumQ - 1) / (kTileM * kNumQ);
        grid = dim3(tiles, p.pair_heads ? p.Hq / kNumQ : p.Hq, p.nseq);
    } else {
        const int nch = (p.max_selected + kTileM - 1) / kTileM;
        grid = p.pair_heads ? dim3(p.Hq / kNumQ, nch, p.nseq)
                            : dim3(p.Hq, (nch + kNumQ - 1) / kNumQ, p.nseq);
    }
    if (grid.x == 0 || grid.y == 0 || grid.z == 0) return cudaSuccess;
    if (d == 64)
        return mode == kModeLocal ? launch_one<64, kModeLocal>(p, grid, stream)
                                  : launch_one<64, kModeGlobal>(p, grid, stream);
    return mode == kModeLocal ? launch_one<128, kModeLocal>(p, grid, stream)
                              : launch_one<128, kModeGlobal>(p, grid, stream);
}

// ---------------------------------------------------------------- timeout probe

__global__ void timeout_probe_kernel(uint32_t* status, unsigned long long limit_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // nothing ever arrives
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
}

cudaError_t launch_timeout_probe(uint32_t* status, unsigned long long limit_ns, cudaStream_t stream)
{
    timeout_probe_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace logo

