// attn_prefix.cu -- B200 (sm_100a) prefix-masked attention forward: kernels and C ABI.
//
// The operation (declared in include/attn_prefix.h) is scaled-dot-product attention in
// which batch element b sees only its first kv_len[b] keys.  That is the boolean
// [B,1,1,Tk] key-prefix mask of "Rewrite prefix key-padding masks as k/v truncation to
// keep SDPA on the flash path" ("Problem", "Fix"), which equals truncating k/v to the
// valid rows, carried as a per-batch count like the key_value_seq_lengths of "Add
// sequence-parallel multi-GPU inference ... and a cuDNN flash attention option" ("cuDNN
// flash attention").  The softmax is an fp32 online softmax that also emits the per-row
// log-sum-exp, so partial results over key chunks combine exactly ("Sequence-parallel
// inference" on the same page): attn_prefix_fwd_split + attn_lse_combine.
//
// Kernels in this file (the CTA-pair kernel for head dims 128 and 256 is in
// pair_kernel.cuh, the multi-range key gather in segments.cuh):
//
// attn_fwd_kernel<D, SPLIT>: one CTA = one 128-row query tile of one (b, h), optionally
// one key chunk.  Roles:
//   producer warp   TMA: Q tile once, then K and V chunks into a ring of 16 KB shared-
//                   memory slots, in exactly the order the MMA thread consumes them.  Key
//                   tiles at or beyond kv_len are never requested.
//   MMA warp        one thread: S_j = Q K_j^T with both operands in shared memory into a
//                   double-buffered fp32 TMEM tile (128 x 128), and O += P_j V_j with P
//                   read from TMEM and V from shared memory into an fp32 TMEM
//                   accumulator (128 x D).  It also owns the TMEM allocation.
//   relay warp      performs the blocking mbarrier waits in the MMA thread's order and
//                   publishes a count of completed events, which the MMA thread polls.
//   softmax warps   thread = query row = TMEM lane.  Scores of keys >= kv_len are
//                   replaced by -inf by selection; the running max is kept in the log2
//                   domain and O is rescaled in TMEM only when the max grows by more than
//                   2^8 (exact either way: O and the row sum always share one reference
//                   max).  At the end O is divided by the row sum and written as bf16
//                   (fp32 for split partials) with lse = ln(sum) + max.
// Head dims 32 and 64 run in two-group mode (two softmax warpgroups on alternate key
// tiles, each with its own O accumulator and P buffer in TMEM, S issued ahead of PV, an
// exact log-sum-exp merge at the end; 352 threads).  The two warps that share a
// sub-partition run their exponentials whenever their tiles are ready: the MUFU serves
// both, and neither waits for the other (turns taken in tile order cost 7 % against
// this on B200, once the MMA warp issued converged and stopped spinning).  Head
// dims 128 and 256 (test hook only) use one softmax warpgroup that stores P over S (224
// threads).
// lse_combine_kernel<D>: the exact log-sum-exp combination of split partials, one warp
// per output row (also run inside the split kernels when the combine is fused).
//
// The last, partial key tile of a range is read as the window [k_end - 128, k_end): every
// row copied is a valid key (or a zero-filled row at a negative coordinate) and the
// columns that belong to earlier tiles are masked by selection, so key padding (NaN
// included) is never even read.
//
// Every mbarrier wait is bounded (%globaltimer); on expiry the CTA raises a sticky
// device flag, drains its copies and MMAs in flight, frees its TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "attn_prefix.h"
#include "ptx.cuh"
#include "tmem_ops.cuh"
#include "softmax_math.cuh"

namespace attn {

constexpr int BM = 128;               // query rows per CTA (one TMEM lane each)
constexpr int BN = 128;               // keys per tile
constexpr int SMEM_LIMIT = 232448;    // 227 KB opt-in dynamic shared memory per block
constexpr uint32_t TMEM_COLS = 512;   // S0 [0,128) S1 [128,256) O [256, 256+D)
constexpr uint32_t O_COL = 256;
constexpr float RESCALE_LOG2 = 8.0f;  // rescale O only when the max grows by > 2^8
constexpr uint32_t XCH_ID = 9;     // named barrier: the two softmax groups' epilogue exchange
constexpr float LN2 = 0.69314718055994530942f;
constexpr float LOG2E = 1.44269504088896340736f;

constexpr unsigned STATUS_TIMEOUT = 1u;
constexpr unsigned STATUS_KVLEN = 2u;
constexpr unsigned STATUS_LAYOUT = 4u;   // dynamic shared memory not 1024-byte aligned

template <int D>
struct Cfg {
    static constexpr int SW = (D >= 64) ? 128 : 64;   // swizzle span in bytes
    static constexpr int BLK = SW / 2;                // bf16 columns per swizzle block
    static constexpr int NBLK = D / BLK;              // column blocks per row
    static constexpr int Q_BYTES = BM * D * 2;
    static constexpr int SLOT = BN * SW;              // bytes of one K chunk == one V chunk
    static constexpr int KCH = NBLK;                  // K tile: one chunk per column block
    static constexpr int VCH = NBLK;                  // V tile: chunks of V_ROWS key rows
    static constexpr int V_ROWS = BN / VCH;
    // Head dims whose two O accumulators and two P buffers fit in TMEM beside the two S
    // buffers run two softmax warpgroups (even and odd key tiles) with P kept apart from
    // S; larger ones run one warpgroup with P stored over S.
    static constexpr bool DUAL = O_COL + 2 * D + BN <= TMEM_COLS;
    static constexpr uint32_t P_COL = O_COL + 2 * D;    // DUAL: P_w at P_COL + w * BN/2
    static constexpr int SM_WARPS = DUAL ? 8 : 4;
    static constexpr int WARP_PROD = SM_WARPS;          // TMA producer
    static constexpr int WARP_MMA = SM_WARPS + 1;       // MMA issuer, TMEM owner
    static constexpr int WARP_RELAY = SM_WARPS + 2;     // wait relay
    static constexpr int THREADS = 32 * (SM_WARPS + 3);
    static constexpr int XCH_BYTES = DUAL ? 2 * 2 * BM * 4 : 0;   // per-group (max, sum) exchange
    static constexpr int NSLOTS_RAW = (SMEM_LIMIT - Q_BYTES - 2048 - XCH_BYTES) / SLOT;
    static constexpr int GRP = (KCH >= 2) ? 2 : 1;      // chunks per ring group (one barrier pair)
    static constexpr int NSLOTS_CAP = NSLOTS_RAW > 16 ? 16 : NSLOTS_RAW;
    static constexpr int NSLOTS = NSLOTS_CAP / GRP * GRP;
    static constexpr int NG = NSLOTS / GRP;             // ring groups
    static constexpr int SMEM_BYTES = 1024 + Q_BYTES + NSLOTS * SLOT + 1024 + XCH_BYTES;
    static constexpr uint32_t LAYOUT = (SW == 128) ? 2u : 4u;
    static_assert(D % BLK == 0, "head dim must be a multiple of the swizzle block");
    static_assert(V_ROWS % 16 == 0, "value chunks must hold whole 16-key MMA steps");
    static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory budget");
    static_assert(O_COL + D <= TMEM_COLS, "TMEM budget");
    static_assert(KCH % GRP == 0 && VCH % GRP == 0 && NG <= 16, "ring grouping");
};

// Barrier slots inside the shared-memory control block.
enum : int {
    BAR_Q = 0,
    BAR_FULL = 1,       // [16] ring group filled (TMA tx)
    BAR_EMPTY = 17,     // [16] ring group consumed (tcgen05.commit)
    BAR_S = 33,         // [2] S_j ready in TMEM buffer j&1
    BAR_P = 35,         // [2] P_j stored over S_j (one arrival per softmax warp of its group)
    BAR_PVD = 37,       // [2] PV into accumulator O_w complete (one phase per PV)
    BAR_DRAIN = 39,
    BAR_SC = 40,        // [2] two-group mode: S_j read out of TMEM buffer j&1 (one arrival per warp)
    BAR_OFIN = 42,      // the last PV complete (completes once; its commit covers every MMA)
    NUM_BARS = 43
};

struct Params {
    const int32_t* kv_len;
    __nv_bfloat16* out;   // single pass, or split with fused combine: bf16 [B,H,Tq,D] at strides out_s*
    float* lse;           // single pass, or split with fused combine: fp32 [B,H,Tq] or null
    float* part_out;      // split: fp32 [C,B,H,Tq,D]
    float* part_lse;      // split: fp32 [C,B,H,Tq]
    int* counters;        // split with fused combine: int32 [B*H*ceil(Tq/128)], else null
    long long out_sb, out_sh, out_st;   // element strides of out along b, h, t (d contiguous)
    int B, H, Tq, Tk;
    int n_qtiles;
    int num_splits;
    int chunk_len;        // keys per split chunk (multiple of BN)
    float scale_log2;     // scale * log2(e)
    unsigned long long wait_ns;
    unsigned debug;
};

__device__ unsigned int g_attn_status = 0;

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Bounded wait on an mbarrier phase.  Returns false if the CTA's abort flag is set or
// the time limit runs out (which sets the abort flag and the device timeout flag).
__device__ __noinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                      unsigned long long limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > limit_ns) {
            *abort_flag = 1;
            atomicOr(&g_attn_status, STATUS_TIMEOUT);
            return false;
        }
    }
}

// Bounded wait that ignores the abort flag: used only to drain work already in flight.
__device__ __noinline__ bool wait_bar_drain(uint32_t bar, uint32_t parity,
                                            unsigned long long limit_ns) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns) {
            atomicOr(&g_attn_status, STATUS_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Exact combination of one row's split partials, by one warp (lane = thread % 32):
//   M = max_c lse_c,  lse = M + ln sum_c exp(lse_c - M),  out = sum_c exp(lse_c - lse) O_c,
// the log-sum-exp rule of split-KV; a row whose every chunk is empty gives 0 / -inf.
// Partials are [C][rows][D] and [C][rows]; out_row points at the row's D outputs, lse
// is indexed by row.  FRESH: the partials were written by other
// CTAs of the running kernel, so they are read through L2 (ld.global.cg) instead of the
// read-only path; the arithmetic, and so the result, is the same either way.
template <typename T, bool FRESH>
__device__ __forceinline__ T ld_part(const T* ptr) {
    if constexpr (FRESH) return __ldcg(ptr);
    else return __ldg(ptr);
}
template <int D, bool FRESH>
__device__ __forceinline__ void combine_row(const float* __restrict__ part_out, const float* __restrict__ part_lse,
                                            int C, long long rows, long long row, __nv_bfloat16* __restrict__ out_row,
                                            float* __restrict__ lse, int lane) {
    constexpr int PER = D / 32;
    float M = -INFINITY;
    for (int c = lane; c < C; c += 32) M = fmaxf(M, ld_part<float, FRESH>(part_lse + c * rows + row));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.0f;
    float L = -INFINITY;
    if (M != -INFINITY) {
        float s = 0.0f;
        for (int c = lane; c < C; c += 32) s += expf(ld_part<float, FRESH>(part_lse + c * rows + row) - M);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        L = M + logf(s);
        // Chunk weights 32 at a time, one per lane, broadcast by shuffle: the partial loads
        // of consecutive chunks then depend on nothing loaded in the loop and overlap.  An
        // empty chunk (lse_c = -inf, partial stored as zeros) has weight 0 and adds 0.
        for (int cb = 0; cb < C; cb += 32) {
            const int c_l = cb + lane;
            const float w_l = c_l < C ? expf(ld_part<float, FRESH>(part_lse + c_l * rows + row) - L) : 0.0f;
            const int nc = min(32, C - cb);
#pragma unroll 4
            for (int t = 0; t < nc; ++t) {
                const float w = __shfl_sync(0xffffffffu, w_l, t);
                const float* src = part_out + (static_cast<long long>(cb + t) * rows + row) * D + lane * PER;
                if constexpr (PER % 4 == 0) {
#pragma unroll
                    for (int e = 0; e < PER; e += 4) {
                        const float4 v4 = ld_part<float4, FRESH>(reinterpret_cast<const float4*>(src + e));
                        acc[e] += w * v4.x;
                        acc[e + 1] += w * v4.y;
                        acc[e + 2] += w * v4.z;
                        acc[e + 3] += w * v4.w;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < PER; ++e) acc[e] += w * ld_part<float, FRESH>(src + e);
                }
            }
        }
    }
    __nv_bfloat16* dst = out_row + lane * PER;
    if constexpr (PER == 1) {
        dst[0] = __float2bfloat16_rn(acc[0]);
    } else {
#pragma unroll
        for (int e = 0; e < PER; e += 2) *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(acc[e], acc[e + 1]);
    }
    if (lane == 0 && lse != nullptr) lse[row] = L;
}

// Split-KV with the combine fused in: called by all `nthreads` threads of a CTA (thread
// index `t`) at its very end, once its partials for query rows [q0, q0 + 128) are stored.  Every CTA of every chunk counts itself in on the tile's counter; the
// one that completes the count (the last chunk to finish, in whatever order) combines
// the tile's rows from all chunks' partials into p.out / p.lse and zeroes the counter
// for the next call.  This is the "only softmax statistics cross" combine of split-KV
// without a second launch or a second pass over the partials from DRAM.  The count is
// taken even after an abort, so the counters always return to zero.
template <int D>
__device__ __forceinline__ void fused_combine_tail(const Params& p, int bh, int q0, int t, int nthreads,
                                                   volatile int* flag) {
    if (q0 >= p.Tq) return;   // a pair's second tile past the last query row: no rows
    __threadfence();          // this thread's partial stores, visible device-wide
    __syncthreads();
    const long long tile = static_cast<long long>(bh) * ((p.Tq + BM - 1) / BM) + q0 / BM;
    if (t == 0) {
        const int last = atomicAdd(p.counters + tile, 1) == p.num_splits - 1;
        if (last) p.counters[tile] = 0;
        *flag = last;
    }
    __syncthreads();
    if (!*flag) return;
    __threadfence();          // the other chunks' partials, counted in before the count completed
    const long long rows = static_cast<long long>(p.B) * p.H * p.Tq;
    const int nr = min(BM, p.Tq - q0);
    const int b = bh / p.H, h = bh - b * p.H;
    for (int r = t >> 5; r < nr; r += nthreads >> 5)
        combine_row<D, true>(p.part_out, p.part_lse, p.num_splits, rows, static_cast<long long>(bh) * p.Tq + q0 + r,
                             p.out + b * p.out_sb + h * p.out_sh + (q0 + r) * p.out_st, p.lse, t & 31);
}

template <int D, bool SPLIT>
__global__ void __launch_bounds__(Cfg<D>::THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const Params p) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sQ = smem;
    uint8_t* sKV = smem + C::Q_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + C::NSLOTS * C::SLOT);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    uint32_t* ready_seq = tmem_holder + 2;   // events the relay warp has seen complete
    const uint32_t ready_addr = smem_u32(ready_seq);
    const uint32_t bar0 = smem_u32(bars);
    const uint32_t sQ_addr = smem_u32(sQ);
    const uint32_t sKV_addr = smem_u32(sKV);
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // ---- work unit: query tile fastest, then split chunk, then (b, h)
    int unit = blockIdx.x;
    const int qtile = unit % p.n_qtiles;
    unit /= p.n_qtiles;
    const int split = SPLIT ? unit % p.num_splits : 0;
    const int bh = SPLIT ? unit / p.num_splits : unit;
    const int b = bh / p.H;
    const int h = bh - b * p.H;
    const int q0 = qtile * BM;

    int kv = __ldg(p.kv_len + b);
    if (kv < 0 || kv > p.Tk) {
        if (tid == 0) atomicOr(&g_attn_status, STATUS_KVLEN);
        kv = kv < 0 ? 0 : p.Tk;
    }
    const int k_begin = SPLIT ? split * p.chunk_len : 0;
    const int k_end = SPLIT ? min(kv, k_begin + p.chunk_len) : kv;
    const int n_tiles = (k_end > k_begin) ? (k_end - k_begin + BN - 1) / BN : 0;
    // The last, partial tile is read as the window [k_end - BN, k_end); its leading
    // last_lo columns belong to earlier tiles (or precede the range) and are masked.
    const int last_lo = n_tiles > 0 ? n_tiles * BN - (k_end - k_begin) : 0;
    auto tile_key0 = [&](int j) { return (j == n_tiles - 1 && last_lo > 0) ? k_end - BN : k_begin + j * BN; };

    if (tid == 0) {
        mbar_init(BAR(BAR_Q), 1);
        for (int g = 0; g < C::NG; ++g) {
            mbar_init(BAR(BAR_FULL + g), 1);
            mbar_init(BAR(BAR_EMPTY + g), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(BAR(BAR_S + i), 1);
            mbar_init(BAR(BAR_P + i), 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(BAR(BAR_PVD + i), 1);
            mbar_init(BAR(BAR_SC + i), 4);
        }
        mbar_init(BAR(BAR_DRAIN), 1);
        mbar_init(BAR(BAR_OFIN), 1);
        *abort_flag = 0;
        *ready_seq = 0u;
        fence_mbar_init();
    }
    if (warp == C::WARP_MMA) {
        tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const unsigned long long wlim = p.wait_ns;

    if (warp == C::WARP_PROD) {
        // ================================================================ producer
        // Loads go out in the order the MMA thread consumes them: K_0, K_1, then
        // V_j, K_{j+2} for every tile j (two-group mode: K_2, then K_{j+3}, V_j).  Each tile half is GRP-chunk groups; one ring
        // group (GRP consecutive 16 KB slots) has one full and one empty barrier.
        if (lane == 0 && n_tiles > 0) {
            tma_prefetch_map(&tm_q);
            tma_prefetch_map(&tm_k);
            tma_prefetch_map(&tm_v);
            mbar_arrive_expect_tx(BAR(BAR_Q), C::Q_BYTES);
#pragma unroll
            for (int blk = 0; blk < C::NBLK; ++blk)
                tma_load_4d(sQ_addr + blk * BM * C::SW, &tm_q, blk * C::BLK, q0, h, b, BAR(BAR_Q));

            int gi = 0;
            uint32_t phase = 0;
            uint32_t pending = 0, pend_parity = 0;   // per ring group: fill issued, its parity
            int dropped = -1;
            bool ok = true;
            auto acquire = [&]() -> bool {
                ok = wait_bar(BAR(BAR_EMPTY + gi), phase ^ 1u, abort_flag, wlim);
                if (ok) mbar_arrive_expect_tx(BAR(BAR_FULL + gi), C::GRP * C::SLOT);
                return ok;
            };
            auto release_slot_bookkeeping = [&]() {
                pending |= 1u << gi;
                pend_parity = (pend_parity & ~(1u << gi)) | (phase << gi);
                if (++gi == C::NG) {
                    gi = 0;
                    phase ^= 1u;
                }
            };
            auto load_k = [&](int j) {
                const int key0 = tile_key0(j);
#pragma unroll 1
                for (int g = 0; g < C::KCH / C::GRP && ok; ++g) {
                    if (!acquire()) break;
#pragma unroll
                    for (int cc = 0; cc < C::GRP; ++cc) {
                        const int c = g * C::GRP + cc;
                        if ((p.debug & ATTN_DEBUG_DROP_COPY) && j == 0 && c == 0) {
                            dropped = gi;   // announced, never issued: the consumer's wait runs out
                            continue;
                        }
                        tma_load_4d(sKV_addr + (gi * C::GRP + cc) * C::SLOT, &tm_k, c * C::BLK, key0, h, b,
                                    BAR(BAR_FULL + gi));
                    }
                    release_slot_bookkeeping();
                }
            };
            auto load_v = [&](int j) {
                const int key0 = tile_key0(j);
#pragma unroll 1
                for (int g = 0; g < C::VCH / C::GRP && ok; ++g) {
                    if (!acquire()) break;
#pragma unroll
                    for (int cc = 0; cc < C::GRP; ++cc) {
                        const int c = g * C::GRP + cc;
#pragma unroll
                        for (int blk = 0; blk < C::NBLK; ++blk)
                            tma_load_4d(sKV_addr + (gi * C::GRP + cc) * C::SLOT + blk * C::V_ROWS * C::SW, &tm_v,
                                        blk * C::BLK, key0 + c * C::V_ROWS, h, b, BAR(BAR_FULL + gi));
                    }
                    release_slot_bookkeeping();
                }
            };
            load_k(0);
            if (n_tiles > 1) load_k(1);
            if constexpr (C::DUAL) {
                // S runs three tiles ahead of PV: K_2, then K_{j+3}, V_j per tile j
                if (n_tiles > 2) load_k(2);
#pragma unroll 1
                for (int j = 0; j < n_tiles && ok; ++j) {
                    if (j + 3 < n_tiles) load_k(j + 3);
                    load_v(j);
                }
            } else {
#pragma unroll 1
                for (int j = 0; j < n_tiles && ok; ++j) {
                    load_v(j);
                    if (j + 2 < n_tiles) load_k(j + 2);
                }
            }
            if (!ok) {
                // Drain: every copy issued must land before this CTA's memory is reused.
                wait_bar_drain(BAR(BAR_Q), 0, wlim);
                for (int g = 0; g < C::NG; ++g)
                    if (((pending >> g) & 1u) && g != dropped)
                        wait_bar_drain(BAR(BAR_FULL + g), (pend_parity >> g) & 1u, wlim);
            }
        }
        __syncwarp();
    } else if (warp == C::WARP_MMA) {
        // ================================================================ MMA issuer (one warp)
        // Two readiness events per tile, published by the relay warp: "P_j stored and
        // V_j landed" and "K_{j+2} landed" (two-group mode: "S_{j+1} read out and K_{j+3}
        // landed" and "V_j landed", and this warp waits for "P_j stored" itself, with a
        // suspending try_wait: the relay's wake-up and this warp's poll had put ~850
        // cycles between the last P arrival and PV_j; same-box A/B +4.5 % at N 13622 and
        // 7784, +2.2 % at N 31136).  Between them the 8 PV and 16 S MMAs of a
        // tile are issued as straight-line code from precomputed descriptors, so the
        // tensor pipe's queue stays fed (the tile's MMA mix alone runs at the tensor
        // peak; the issuing code's overhead is what decides the rate).  The whole warp
        // runs it converged and its elected lane issues, so the descriptors stay
        // warp-uniform; every wait decision is lane 0's, broadcast.
        if (n_tiles > 0) {
            constexpr uint32_t IDESC_S = make_idesc_bf16(BM, BN, false);
            constexpr uint32_t IDESC_PV = make_idesc_bf16(BM, D, true);
            constexpr int KG = C::KCH / C::GRP;
            constexpr int VG = C::VCH / C::GRP;
            constexpr uint32_t GSTEP = static_cast<uint32_t>((C::GRP * C::SLOT) >> 4);   // per ring group
            // Descriptor templates; the 14-bit address field is advanced by plain adds.
            const uint64_t q_desc0 = make_smem_desc(sQ_addr, 16, 8 * C::SW, C::LAYOUT);
            const uint64_t k_desc0 = make_smem_desc(sKV_addr, 16, 8 * C::SW, C::LAYOUT);
            const uint64_t v_desc0 = make_smem_desc(sKV_addr, C::V_ROWS * C::SW, 8 * C::SW, C::LAYOUT);
            int gi = 0;   // ring group of the next K/V group to consume
            uint32_t consumed = 0;
            bool ok = __all_sync(0xffffffffu, wait_bar(BAR(BAR_Q), 0, abort_flag, wlim));
            auto ring = [&](int g) { return (gi + g < C::NG) ? gi + g : gi + g - C::NG; };
            auto advance = [&](int n) { gi = (gi + n < C::NG) ? gi + n : gi + n - C::NG; };
            // The relay warp performs the blocking mbarrier waits in this thread's order
            // and publishes how many events have completed; polling that word costs a
            // shared-memory load instead of an mbarrier round trip.
            // lane 0 reads the relay's count and broadcasts it (one shared-memory load per poll)
            auto poll_word = [&](uint32_t addr) -> uint32_t {
                uint32_t v = 0;
                if (lane == 0) v = ld_acquire_smem(addr);
                return __shfl_sync(0xffffffffu, v, 0);
            };
            auto next_event = [&]() -> bool {
                ++consumed;
                bool ok_ev = true;
                if (poll_word(ready_addr) < consumed) {
                    const uint64_t t0 = global_timer_ns();
                    while (true) {
                        __nanosleep(32);   // a spinning poll takes issue slots from the softmax warps beside it
                        if (poll_word(ready_addr) >= consumed) break;
                        if (*abort_flag) {
                            ok_ev = false;
                            break;
                        }
                        if (global_timer_ns() - t0 > wlim) {
                            if (lane == 0) {
                                *abort_flag = 1;
                                atomicOr(&g_attn_status, STATUS_TIMEOUT);
                            }
                            ok_ev = false;
                            break;
                        }
                    }
                }
                return __shfl_sync(0xffffffffu, ok_ev ? 1 : 0, 0) != 0;
            };
            auto uniform = [&](bool v) { return __shfl_sync(0xffffffffu, v ? 1 : 0, 0) != 0; };
            // a barrier the softmax warps arrive on, waited with try_wait (suspends the warp)
            auto wait_arrivals = [&](uint32_t bar, uint32_t par) -> bool {
                if (uniform(mbar_try_wait(bar, par))) return true;
                const uint64_t t0 = global_timer_ns();
                while (true) {
                    if (uniform(mbar_try_wait(bar, par))) return true;
                    if (uniform(*abort_flag != 0)) return false;
                    if (uniform(global_timer_ns() - t0 > wlim)) {
                        if (lane == 0) {
                            *abort_flag = 1;
                            atomicOr(&g_attn_status, STATUS_TIMEOUT);
                        }
                        return false;
                    }
                }
            };
            auto issue_s = [&](int j) {
                const uint32_t d_tmem = tmem + static_cast<uint32_t>(j & 1) * BN;
#pragma unroll
                for (int g = 0; g < KG; ++g) {
                    const uint64_t kd = k_desc0 + static_cast<uint64_t>(ring(g)) * GSTEP;
#pragma unroll
                    for (int cc = 0; cc < C::GRP; ++cc) {
                        const int c = g * C::GRP + cc;
#pragma unroll
                        for (int kk = 0; kk < C::BLK / 16; ++kk)
                            mma_ss_elect(d_tmem, q_desc0 + static_cast<uint64_t>(((c * BM * C::SW) >> 4) + kk * 2),
                                   kd + static_cast<uint64_t>(((cc * C::SLOT) >> 4) + kk * 2), IDESC_S,
                                   (c | kk) != 0 ? 1u : 0u);
                    }
                }
#pragma unroll
                for (int g = 0; g < KG; ++g) tc_commit_elect(BAR(BAR_EMPTY + ring(g)));
                tc_commit_elect(BAR(BAR_S + (j & 1)));
                advance(KG);
            };
            auto issue_pv = [&](int j) {
                // Every 16-key step is issued, partial last tile included: its masked
                // columns hold P = 0 against value rows that are valid keys of earlier
                // tiles (or zero fill), never padding.
                // Two-group mode: PV_j reads P_{j&1} and adds into O_{j&1}; each starts fresh.
                const uint32_t p_tmem = C::DUAL ? tmem + C::P_COL + static_cast<uint32_t>(j & 1) * (BN / 2)
                                                : tmem + static_cast<uint32_t>(j & 1) * BN;
                const uint32_t o_tmem = tmem + O_COL + (C::DUAL ? static_cast<uint32_t>((j & 1) * D) : 0u);
                const uint32_t acc0 = (j < (C::DUAL ? 2 : 1)) ? 0u : 1u;
#pragma unroll
                for (int g = 0; g < VG; ++g) {
                    const uint64_t vd = v_desc0 + static_cast<uint64_t>(ring(g)) * GSTEP;
#pragma unroll
                    for (int cc = 0; cc < C::GRP; ++cc) {
#pragma unroll
                        for (int kk = 0; kk < C::V_ROWS / 16; ++kk) {
                            const int kb = (g * C::GRP + cc) * (C::V_ROWS / 16) + kk;
                            mma_ts_elect(o_tmem, p_tmem + static_cast<uint32_t>(kb) * 8u,
                                   vd + static_cast<uint64_t>(((cc * C::SLOT) >> 4) + ((kk * 16 * C::SW) >> 4)),
                                   IDESC_PV, kb == 0 ? acc0 : 1u);
                        }
                    }
                }
#pragma unroll
                for (int g = 0; g < VG; ++g) tc_commit_elect(BAR(BAR_EMPTY + ring(g)));
                // One phase per PV on the accumulator's barrier: the softmax group waits
                // it before rescaling O or reusing the P buffer, the epilogue before reading.
                tc_commit_elect(BAR(BAR_PVD + (C::DUAL ? (j & 1) : 0)));
                if (j == n_tiles - 1) tc_commit_elect(BAR(BAR_OFIN));
                advance(VG);
            };
            if (ok) ok = next_event();
            if (ok) {
                tc_fence_after();
                issue_s(0);
            }
            if (ok && n_tiles > 1) {
                ok = next_event();
                if (ok) {
                    tc_fence_after();
                    issue_s(1);
                }
            }
            if constexpr (C::DUAL) {
                // P has its own buffers, so S_{j+2} may overwrite S_j as soon as the group
                // has read it out: S runs ahead of PV (S_2, then S_{j+3} before PV_j).
                if (ok && n_tiles > 2) {
                    ok = next_event();   // S_0 read out and K_2 landed
                    if (ok) {
                        tc_fence_after();
                        issue_s(2);
                    }
                }
#pragma unroll 1
                for (int j = 0; j < n_tiles && ok; ++j) {
                    if (j + 3 < n_tiles) {
                        ok = next_event();   // S_{j+1} read out and K_{j+3} landed
                        if (!ok) break;
                        tc_fence_after();
                        issue_s(j + 3);
                    }
                    ok = next_event();   // V_j landed
                    if (!ok) break;
                    ok = wait_arrivals(BAR(BAR_P + (j & 1)), (j >> 1) & 1);   // P_j stored
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(j);
                }
            } else {
#pragma unroll 1
                for (int j = 0; j < n_tiles && ok; ++j) {
                    ok = next_event();   // P_j stored and V_j landed
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(j);
                    if (j + 2 < n_tiles) {
                        ok = next_event();   // K_{j+2} landed
                        if (!ok) break;
                        tc_fence_after();
                        issue_s(j + 2);
                    }
                }
            }
            // Drain: every MMA issued completes before TMEM is released.
            tc_commit_elect(BAR(BAR_DRAIN));
            __syncwarp();
            wait_bar_drain(BAR(BAR_DRAIN), 0, wlim);
        }
        __syncwarp();
    } else if (warp == C::WARP_RELAY) {
        // ================================================================ wait relay
        // Waits on the ring groups and P barriers in the MMA thread's consumption order
        // and publishes one completed event per MMA batch with a release store: K_0,
        // K_1, then per tile j "P_j + V_j" and "K_{j+2}"; the MMA thread acquires it.
        // Two-group mode: K_0, K_1, "S_0 read + K_2", then per tile j "S_{j+1} read +
        // K_{j+3}" and "V_j" (the MMA thread waits for P_j itself).
        if (lane == 0 && n_tiles > 0) {
            int gi = 0;
            uint32_t phase = 0, seq = 0;
            bool ok = true;
            auto group = [&]() {
                ok = ok && wait_bar(BAR(BAR_FULL + gi), phase, abort_flag, wlim);
                if (++gi == C::NG) {
                    gi = 0;
                    phase ^= 1u;
                }
            };
            auto publish = [&]() {
                if (ok) st_release_smem(ready_addr, ++seq);
            };
            auto relay_s = [&]() {
                for (int g = 0; g < C::KCH / C::GRP; ++g) group();
                publish();
            };
            relay_s();
            if (n_tiles > 1) relay_s();
            if constexpr (C::DUAL) {
                auto s_read = [&](int t) {
                    ok = ok && wait_bar(BAR(BAR_SC + (t & 1)), (t >> 1) & 1, abort_flag, wlim);
                };
                if (n_tiles > 2) {
                    s_read(0);
                    relay_s();
                }
#pragma unroll 1
                for (int j = 0; j < n_tiles && ok; ++j) {
                    if (j + 3 < n_tiles) {
                        s_read(j + 1);
                        relay_s();
                    }
                    for (int g = 0; g < C::VCH / C::GRP; ++g) group();   // V_j
                    publish();
                }
            } else {
#pragma unroll 1
                for (int j = 0; j < n_tiles && ok; ++j) {
                    for (int g = 0; g < C::VCH / C::GRP; ++g) group();   // V_j first: usually landed
                    ok = ok && wait_bar(BAR(BAR_P + (j & 1)), (j >> 1) & 1, abort_flag, wlim);
                    publish();
                    if (j + 2 < n_tiles) relay_s();
                }
            }
        }
        __syncwarp();
    } else {
        // ================================================================ softmax
        // Thread t of warpgroup w (warps 4w .. 4w+3) owns query row r = t % 128 (TMEM lane r).
        // Two-group mode (head dims up to 64): warpgroup w takes the key tiles j = w (mod 2)
        // with its own running max, row sum, O accumulator O_w and P buffer P_w, so one
        // group's exponentials overlap the other's MMA round trip; the two partial results
        // are combined exactly at the end (the log-sum-exp rule of split-KV).  Otherwise one
        // warpgroup takes every tile and stores P over S.
        constexpr bool DUAL = C::DUAL;
        const int wg = warp >> 2;
        const int r = tid & 127;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t o_col = O_COL + (DUAL ? static_cast<uint32_t>(wg * D) : 0u);
        const float sl2 = p.scale_log2;
        const bool pos_scale = sl2 > 0.0f;
        float m_ref = -INFINITY;   // reference max of this group's tiles, log2 domain
        float l_sum = 0.0f;        // row sum relative to m_ref
        bool ok = true;
        const int j0 = DUAL ? wg : 0;
        const int jstep = DUAL ? 2 : 1;
        int seen = 0;              // tiles this group has processed
        // One arrival per warp once its tcgen05 accesses are complete.
        auto warp_arrive = [&](uint32_t bar) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
        };
#pragma unroll 1
        for (int j = j0; j < n_tiles; j += jstep) {
            if (ok) ok = __all_sync(0xffffffffu, wait_bar(BAR(BAR_S + (j & 1)), (j >> 1) & 1, abort_flag, wlim));
            if (!ok) break;
            tc_fence_after();
            const uint32_t s_addr = tmem + lane_base + static_cast<uint32_t>(j & 1) * BN;
            uint32_t raw[BN];
            tmem_ld128_wait(s_addr, raw);
            if constexpr (DUAL) warp_arrive(BAR(BAR_SC + (j & 1)));   // S buffer free for S_{j+2}
            float x[BN];
            const int lo = (j == n_tiles - 1) ? last_lo : 0;   // columns [0, lo) are not this tile's keys
            if (lo > 0) {
#pragma unroll
                for (int c = 0; c < BN; ++c) x[c] = (c >= lo) ? __uint_as_float(raw[c]) : -INFINITY;
            } else {
#pragma unroll
                for (int c = 0; c < BN; ++c) x[c] = __uint_as_float(raw[c]);
            }
            if (!pos_scale) {
                // zero or negative scale: scale every valid score first (the max flips)
#pragma unroll
                for (int c = 0; c < BN; ++c) x[c] = (c >= lo) ? x[c] * sl2 : -INFINITY;
            }
            // row max (three-input maxima)
            const float mx = row_max(x) * (pos_scale ? sl2 : 1.0f);
            float factor = 1.0f;
            bool rescale = false;
            if (seen == 0) {
                m_ref = mx;
            } else if (__any_sync(0xffffffffu, mx > m_ref + RESCALE_LOG2)) {
                const float m_new = fmaxf(m_ref, mx);
                factor = fast_exp2(m_ref - m_new);
                m_ref = m_new;
                rescale = true;
            }
            const float mul = pos_scale ? sl2 : 1.0f;
            const float neg_m = -m_ref;
            if constexpr (DUAL) {
                // PV_{j-2}, this group's previous PV, reads P_w and adds into O_w: it must be
                // complete before P_w is rewritten (P is stored as it is computed, below) and
                // before O_w is rescaled.  The parity wait is unambiguous: the barrier has
                // passed the phase before (waited on this group's previous tile) and cannot
                // pass the one after, whose PV needs this tile's P.
                if (seen > 0) {
                    ok = __all_sync(0xffffffffu,
                                    wait_bar(BAR(BAR_PVD + (j & 1)), (seen - 1) & 1, abort_flag, wlim));
                    if (!ok) break;
                    tc_fence_after();
                }
            }
            // p = 2^(x * mul - m): the scale-and-shift and the row sum in packed pairs; P is
            // stored 32 columns at a time, over S_j (one group) or into P_w (two groups).
            const uint32_t p_addr = DUAL ? tmem + lane_base + C::P_COL + static_cast<uint32_t>(j & 1) * (BN / 2) : s_addr;
            float2 sp[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) sp[t] = make_float2(0.0f, 0.0f);
            const float2 mul_2 = make_float2(mul, mul);
            const float2 neg_m2 = make_float2(neg_m, neg_m);
#pragma unroll
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float2 y = fma2(make_float2(x[cc * 32 + 2 * e], x[cc * 32 + 2 * e + 1]), mul_2, neg_m2);
                    const float p0 = fast_exp2(y.x);
                    const float p1 = fast_exp2(y.y);
                    sp[e & 3] = add2(sp[e & 3], make_float2(p0, p1));
                    pk[e] = pack_bf16x2(p0, p1);
                }
                tmem_st16_at(p_addr + cc * 16, pk);
            }
            const float tile_sum = ((sp[0].x + sp[1].x) + (sp[2].x + sp[3].x)) + ((sp[0].y + sp[1].y) + (sp[2].y + sp[3].y));
            l_sum = l_sum * factor + tile_sum;
            // One group: PV_{j-1} must be complete before O is rescaled.  The parity wait is
            // unambiguous: S_j, issued after PV_{j-2}, is complete, so the barrier has passed
            // the phase before; the phase after needs this tile's P.
            if (!DUAL && seen > 0 && rescale) {
                ok = __all_sync(0xffffffffu, wait_bar(BAR(BAR_PVD), (seen - 1) & 1, abort_flag, wlim));
                if (!ok) break;
                tc_fence_after();
            }
            if (rescale) {
#pragma unroll 1
                for (int oc = 0; oc < D / 32; ++oc) {
                    uint32_t o[32];
                    tmem_ld32_wait(tmem + lane_base + o_col + oc * 32, o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
                    tmem_st32(tmem + lane_base + o_col + oc * 32, o);
                }
            }
            tmem_wait_st();
            warp_arrive(BAR(BAR_P + (j & 1)));
            ++seen;
        }
        // ---- epilogue: the last PV's barrier completes once, after every MMA.  (A parity
        // wait names a phase only while the barrier is at most one phase from it, which
        // the per-PV barriers do not promise here.)
        if (ok && n_tiles > 0) {
            ok = __all_sync(0xffffffffu, wait_bar(BAR(BAR_OFIN), 0, abort_flag, wlim));
            tc_fence_after();
        }
        // combine the groups' partial results: m = max_w m_w, f_w = 2^(m_w - m),
        // l = sum_w l_w f_w, O = sum_w O_w f_w / l (a group with no tile has l_w = 0).
        float f_own = 1.0f, f_other = 0.0f, m_row = m_ref, l_row = l_sum;
        bool other_has = false;
        if constexpr (DUAL) {
            float* xch = reinterpret_cast<float*>(smem + C::Q_BYTES + C::NSLOTS * C::SLOT + 1024);  // [2][2][128]
            xch[(wg * 2 + 0) * 128 + r] = m_ref;
            xch[(wg * 2 + 1) * 128 + r] = l_sum;
            named_barrier_sync(XCH_ID, 256);
            const float m_o = xch[((wg ^ 1) * 2 + 0) * 128 + r];
            const float l_o = xch[((wg ^ 1) * 2 + 1) * 128 + r];
            const bool own_has = l_sum > 0.0f;
            other_has = l_o > 0.0f;
            m_row = own_has ? (other_has ? fmaxf(m_ref, m_o) : m_ref) : m_o;
            f_own = own_has ? fast_exp2(m_ref - m_row) : 0.0f;
            f_other = other_has ? fast_exp2(m_o - m_row) : 0.0f;
            l_row = l_sum * f_own + l_o * f_other;
        }
        const int row = q0 + r;
        const bool in_range = row < p.Tq;
        const bool have = n_tiles > 0;
        const float inv_l = have ? 1.0f / l_row : 0.0f;
        const float lse_val = have ? (m_row + log2f(l_row)) * LN2 : -INFINITY;
        const long long BH = static_cast<long long>(p.B) * p.H;
        const bool own_has_o = DUAL ? (have && l_sum > 0.0f) : have;
        const uint32_t o_col_other = O_COL + static_cast<uint32_t>((wg ^ 1) * D);
        // DUAL: group w writes the 32-column chunks oc = w (mod 2); otherwise group 0 writes all
#pragma unroll 1
        for (int oc = DUAL ? wg : 0; oc < D / 32; oc += DUAL ? 2 : 1) {
            uint32_t o[32];
            if (own_has_o) {
                tmem_ld32_wait(tmem + lane_base + (DUAL ? O_COL + static_cast<uint32_t>(wg * D) : O_COL) + oc * 32, o);
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f_own);
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = 0u;
            }
            if (DUAL && other_has) {
                uint32_t o2[32];
                tmem_ld32_wait(tmem + lane_base + o_col_other + oc * 32, o2);
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    o[e] = __float_as_uint(fmaf(__uint_as_float(o2[e]), f_other, __uint_as_float(o[e])));
            }
            if (!in_range) continue;
            if constexpr (SPLIT) {
                float* dst = p.part_out + ((static_cast<long long>(split) * BH + bh) * p.Tq + row) * D + oc * 32;
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    float4 v4 = make_float4(__uint_as_float(o[e]) * inv_l, __uint_as_float(o[e + 1]) * inv_l,
                                            __uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l);
                    *reinterpret_cast<float4*>(dst + e) = v4;
                }
            } else {
                __nv_bfloat16* dst = p.out + b * p.out_sb + h * p.out_sh + row * p.out_st + oc * 32;
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    uint4 v4;
                    v4.x = pack_bf16x2(__uint_as_float(o[e + 0]) * inv_l, __uint_as_float(o[e + 1]) * inv_l);
                    v4.y = pack_bf16x2(__uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l);
                    v4.z = pack_bf16x2(__uint_as_float(o[e + 4]) * inv_l, __uint_as_float(o[e + 5]) * inv_l);
                    v4.w = pack_bf16x2(__uint_as_float(o[e + 6]) * inv_l, __uint_as_float(o[e + 7]) * inv_l);
                    *reinterpret_cast<uint4*>(dst + e) = v4;
                }
            }
        }
        if (in_range && wg == 0) {
            if constexpr (SPLIT) {
                p.part_lse[(static_cast<long long>(split) * BH + bh) * p.Tq + row] = lse_val;
            } else if (p.lse != nullptr) {
                p.lse[static_cast<long long>(bh) * p.Tq + row] = lse_val;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == C::WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    if constexpr (SPLIT) {
        if (p.counters != nullptr)
            fused_combine_tail<D>(p, bh, q0, tid, C::THREADS, reinterpret_cast<volatile int*>(tmem_holder + 3));
    }
#undef BAR
}

#include "pair_kernel.cuh"

// One warp per output row (see combine_row); out at element strides (sb, sh, st).
template <int D>
__global__ void __launch_bounds__(256) lse_combine_kernel(const float* __restrict__ part_out,
                                                          const float* __restrict__ part_lse, int C,
                                                          long long rows, int H, int Tq,
                                                          __nv_bfloat16* __restrict__ out, long long sb,
                                                          long long sh, long long st, float* __restrict__ lse) {
    const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= rows) return;
    const long long bh = row / Tq, q = row - bh * Tq;
    const long long b = bh / H, h = bh - b * H;
    combine_row<D, false>(part_out, part_lse, C, rows, row, out + b * sb + h * sh + q * st, lse, threadIdx.x & 31);
}

#include "segments.cuh"

}  // namespace attn

// =========================================================================== host side
namespace {

using attn::BM;
using attn::BN;
using attn::Cfg;
using attn::Params;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Test hooks (attn_set_wait_limit_ns, attn_set_debug_flags): process-wide settings read
// by every launch that starts after they are written, from any host thread.
std::atomic<unsigned long long> g_wait_ns{1000000000ull};
std::atomic<unsigned> g_debug{0u};

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Element strides of one [B, H, T, D] operand (d contiguous).
struct Strides {
    long long b, h, t;
};
Strides contiguous(int H, int T, int D) {
    return {static_cast<long long>(H) * T * D, static_cast<long long>(T) * D, static_cast<long long>(D)};
}
// Caller strides, or the contiguous [B,H,T,D] layout for NULL.  Every stride must be a
// non-negative multiple of 8 elements (16-byte rows for TMA and vector stores), and a
// row may not overlap the next one (t >= D).
bool resolve_strides(const attn_strides* in, int H, int T, int D, Strides* out) {
    if (in == nullptr) {
        *out = contiguous(H, T, D);
        return true;
    }
    if (in->b < 0 || in->h < 0 || in->t < D || (in->b & 7) || (in->h & 7) || (in->t & 7)) return false;
    *out = {static_cast<long long>(in->b), static_cast<long long>(in->h), static_cast<long long>(in->t)};
    return true;
}

// Host checks that need no CUDA call.
attn_status check_args(const void* q, const void* k, const void* v, const void* kv_len, const void* out,
                       int B, int H, int Tq, int Tk, int D, float scale) {
    if (!q || !k || !v || !kv_len || !out) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(kv_len) & 3u) != 0) return ATTN_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || Tq <= 0 || Tk <= 0) return ATTN_ERR_INVALID_ARG;
    if (static_cast<long long>(B) * H > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    if (!isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    if (D != 32 && D != 64 && D != 128 && D != 256) return ATTN_ERR_UNSUPPORTED;
    return ATTN_OK;
}

// Device must be compute capability 10.0 (B200 / sm_100a).  Cached per device ordinal
// (0 = not looked up yet, 1 = supported, 2 = not supported); host threads may race on an
// entry, and every one of them writes the same value.
attn_status check_device() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    if (dev < 0 || dev >= 64) return ATTN_ERR_UNSUPPORTED;
    int c = cached[dev].load(std::memory_order_relaxed);
    if (c == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
            cudaGetLastError();
            return ATTN_ERR_CUDA;
        }
        c = (major == 10 && minor == 0) ? 1 : 2;
        cached[dev].store(c, std::memory_order_relaxed);
    }
    return c == 1 ? ATTN_OK : ATTN_ERR_UNSUPPORTED;
}

// A [B, H, T, D] bf16 tensor at element strides s (d contiguous) as a 4-D TMA map with
// dims (D, T, H, B); a box is box_rows rows x box_cols columns of one (b, h).
bool make_map(CUtensorMap* map, const void* base, int B, int H, int T, int D, const Strides& s, int box_cols,
              int box_rows, CUtensorMapSwizzle swz) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(H),
                          static_cast<cuuint64_t>(B)};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(s.t) * 2ull, static_cast<cuuint64_t>(s.h) * 2ull,
                             static_cast<cuuint64_t>(s.b) * 2ull};
    cuuint32_t box[4] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1u, 1u};
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D, bool SPLIT>
attn_status launch_fwd(const void* q, const void* k, const void* v, const Strides* st, Params prm,
                       cudaStream_t stream) {
    using C = Cfg<D>;
    const long long BH = static_cast<long long>(prm.B) * prm.H;
    const CUtensorMapSwizzle swz = (C::SW == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, prm.B, prm.H, prm.Tq, D, st[0], C::BLK, BM, swz) ||
        !make_map(&mk, k, prm.B, prm.H, prm.Tk, D, st[1], C::BLK, BN, swz) ||
        !make_map(&mv, v, prm.B, prm.H, prm.Tk, D, st[2], C::BLK, C::V_ROWS, swz))
        return ATTN_ERR_CUDA;
    const long long grid = static_cast<long long>(prm.n_qtiles) * BH * (SPLIT ? prm.num_splits : 1);
    if (grid > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    auto kern = attn::attn_fwd_kernel<D, SPLIT>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    kern<<<static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, prm);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    return ATTN_OK;
}

// Head dims 128 and 256 run on CTA pairs: 256-row query tiles, each CTA copying half of
// K and V.
template <int D, bool SPLIT>
attn_status launch_fwd_pair(const void* q, const void* k, const void* v, const Strides* st, Params prm,
                            cudaStream_t stream) {
    using C = attn::PairCfg<D>;
    const long long BH = static_cast<long long>(prm.B) * prm.H;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, prm.B, prm.H, prm.Tq, C::D, st[0], 64, C::ROWS, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mk, k, prm.B, prm.H, prm.Tk, C::D, st[1], 64, C::KH, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mv, v, prm.B, prm.H, prm.Tk, C::D, st[2], 64, BN, CU_TENSOR_MAP_SWIZZLE_128B))
        return ATTN_ERR_CUDA;
    prm.n_qtiles = (prm.Tq + 2 * C::ROWS - 1) / (2 * C::ROWS);
    const long long grid = 2LL * prm.n_qtiles * BH * (SPLIT ? prm.num_splits : 1);
    if (grid > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    auto kern = attn::attn_fwd_pair_kernel<D, SPLIT>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    kern<<<static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, prm);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    return ATTN_OK;
}

// st: strides of q, k, v (NULL: all contiguous).
template <bool SPLIT>
attn_status dispatch_fwd(int D, const void* q, const void* k, const void* v, const Params& prm,
                         cudaStream_t stream, const Strides* st = nullptr) {
    Strides dflt[3] = {contiguous(prm.H, prm.Tq, D), contiguous(prm.H, prm.Tk, D), contiguous(prm.H, prm.Tk, D)};
    if (st == nullptr) st = dflt;
    switch (D) {
        case 32: return launch_fwd<32, SPLIT>(q, k, v, st, prm, stream);
        case 64: return launch_fwd<64, SPLIT>(q, k, v, st, prm, stream);
        case 128:
            if (prm.debug & ATTN_DEBUG_SINGLE_CTA) return launch_fwd<128, SPLIT>(q, k, v, st, prm, stream);
            return launch_fwd_pair<128, SPLIT>(q, k, v, st, prm, stream);
        case 256:
            if (prm.debug & ATTN_DEBUG_SINGLE_CTA) return launch_fwd<256, SPLIT>(q, k, v, st, prm, stream);
            return launch_fwd_pair<256, SPLIT>(q, k, v, st, prm, stream);
        default: return ATTN_ERR_UNSUPPORTED;
    }
}

Params base_params(const int32_t* kv_len, int B, int H, int Tq, int Tk, int D, float scale) {
    Params prm;
    memset(&prm, 0, sizeof prm);
    prm.kv_len = kv_len;
    prm.B = B;
    prm.H = H;
    prm.Tq = Tq;
    prm.Tk = Tk;
    prm.n_qtiles = (Tq + BM - 1) / BM;
    prm.num_splits = 1;
    prm.chunk_len = Tk;
    prm.scale_log2 = scale * attn::LOG2E;
    const Strides so = contiguous(H, Tq, D);   // out: contiguous [B,H,Tq,D] unless set otherwise
    prm.out_sb = so.b;
    prm.out_sh = so.h;
    prm.out_st = so.t;
    prm.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
    prm.debug = g_debug.load(std::memory_order_relaxed);
    return prm;
}

}  // namespace

extern "C" {

attn_status attn_prefix_fwd_strided(const void* q, const void* k, const void* v, const int32_t* kv_len, void* out,
                                    float* lse, int B, int H, int Tq, int Tk, int D, float scale,
                                    const attn_strides* q_strides, const attn_strides* k_strides,
                                    const attn_strides* v_strides, const attn_strides* out_strides,
                                    cudaStream_t stream) {
    attn_status st = check_args(q, k, v, kv_len, out, B, H, Tq, Tk, D, scale);
    if (st != ATTN_OK) return st;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_INVALID_ARG;
    Strides s3[3], so;
    if (!resolve_strides(q_strides, H, Tq, D, &s3[0]) || !resolve_strides(k_strides, H, Tk, D, &s3[1]) ||
        !resolve_strides(v_strides, H, Tk, D, &s3[2]) || !resolve_strides(out_strides, H, Tq, D, &so))
        return ATTN_ERR_INVALID_ARG;
    if ((st = check_device()) != ATTN_OK) return st;
    Params prm = base_params(kv_len, B, H, Tq, Tk, D, scale);
    prm.out = static_cast<__nv_bfloat16*>(out);
    prm.lse = lse;
    prm.out_sb = so.b;
    prm.out_sh = so.h;
    prm.out_st = so.t;
    return dispatch_fwd<false>(D, q, k, v, prm, stream, s3);
}

attn_status attn_prefix_fwd(const void* q, const void* k, const void* v, const int32_t* kv_len, void* out,
                            float* lse, int B, int H, int Tq, int Tk, int D, float scale, cudaStream_t stream) {
    return attn_prefix_fwd_strided(q, k, v, kv_len, out, lse, B, H, Tq, Tk, D, scale, nullptr, nullptr, nullptr,
                                   nullptr, stream);
}

int attn_split_chunk_len(int Tk, int num_splits) {
    if (Tk <= 0 || num_splits < 1 || num_splits > 1024) return 0;
    long long per = (static_cast<long long>(Tk) + num_splits - 1) / num_splits;
    per = (per + BN - 1) / BN * BN;
    return static_cast<int>(per);
}

size_t attn_split_lse_offset(int num_splits, int B, int H, int Tq, int D) {
    if (num_splits < 1 || B <= 0 || H <= 0 || Tq <= 0 || D <= 0) return 0;
    size_t o = static_cast<size_t>(num_splits) * B * H * Tq * D * sizeof(float);
    return (o + 255) / 256 * 256;
}

size_t attn_split_workspace_bytes(int num_splits, int B, int H, int Tq, int D) {
    size_t off = attn_split_lse_offset(num_splits, B, H, Tq, D);
    if (off == 0) return 0;
    return off + static_cast<size_t>(num_splits) * B * H * Tq * sizeof(float);
}

attn_status attn_prefix_fwd_split_strided(const void* q, const void* k, const void* v, const int32_t* kv_len,
                                          int num_splits, float* part_out, float* part_lse, int B, int H, int Tq,
                                          int Tk, int D, float scale, const attn_strides* q_strides,
                                          const attn_strides* k_strides, const attn_strides* v_strides,
                                          cudaStream_t stream) {
    attn_status st = check_args(q, k, v, kv_len, part_out, B, H, Tq, Tk, D, scale);
    if (st != ATTN_OK) return st;
    if (!part_lse || (reinterpret_cast<uintptr_t>(part_lse) & 3u)) return ATTN_ERR_INVALID_ARG;
    if (num_splits < 1 || num_splits > 1024) return ATTN_ERR_INVALID_ARG;
    Strides s3[3];
    if (!resolve_strides(q_strides, H, Tq, D, &s3[0]) || !resolve_strides(k_strides, H, Tk, D, &s3[1]) ||
        !resolve_strides(v_strides, H, Tk, D, &s3[2]))
        return ATTN_ERR_INVALID_ARG;
    if ((st = check_device()) != ATTN_OK) return st;
    Params prm = base_params(kv_len, B, H, Tq, Tk, D, scale);
    prm.part_out = part_out;
    prm.part_lse = part_lse;
    prm.num_splits = num_splits;
    prm.chunk_len = attn_split_chunk_len(Tk, num_splits);
    return dispatch_fwd<true>(D, q, k, v, prm, stream, s3);
}

attn_status attn_prefix_fwd_split(const void* q, const void* k, const void* v, const int32_t* kv_len,
                                  int num_splits, float* part_out, float* part_lse, int B, int H, int Tq, int Tk,
                                  int D, float scale, cudaStream_t stream) {
    return attn_prefix_fwd_split_strided(q, k, v, kv_len, num_splits, part_out, part_lse, B, H, Tq, Tk, D, scale,
                                         nullptr, nullptr, nullptr, stream);
}

size_t attn_split_counter_offset(int num_splits, int B, int H, int Tq, int D) {
    const size_t ws = attn_split_workspace_bytes(num_splits, B, H, Tq, D);
    return ws == 0 ? 0 : (ws + 255) / 256 * 256;
}

size_t attn_split_fused_workspace_bytes(int num_splits, int B, int H, int Tq, int D) {
    const size_t off = attn_split_counter_offset(num_splits, B, H, Tq, D);
    if (off == 0) return 0;
    return off + static_cast<size_t>(B) * H * ((static_cast<size_t>(Tq) + BM - 1) / BM) * sizeof(int32_t);
}

attn_status attn_prefix_fwd_split_fused(const void* q, const void* k, const void* v, const int32_t* kv_len,
                                        int num_splits, void* workspace, void* out, float* lse, int B, int H,
                                        int Tq, int Tk, int D, float scale, cudaStream_t stream) {
    attn_status st = check_args(q, k, v, kv_len, out, B, H, Tq, Tk, D, scale);
    if (st != ATTN_OK) return st;
    if (!workspace || !aligned16(workspace) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return ATTN_ERR_INVALID_ARG;
    if (num_splits < 1 || num_splits > 1024) return ATTN_ERR_INVALID_ARG;
    if ((st = check_device()) != ATTN_OK) return st;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    Params prm = base_params(kv_len, B, H, Tq, Tk, D, scale);
    prm.part_out = reinterpret_cast<float*>(ws);
    prm.part_lse = reinterpret_cast<float*>(ws + attn_split_lse_offset(num_splits, B, H, Tq, D));
    prm.counters = reinterpret_cast<int*>(ws + attn_split_counter_offset(num_splits, B, H, Tq, D));
    prm.out = static_cast<__nv_bfloat16*>(out);
    prm.lse = lse;
    prm.num_splits = num_splits;
    prm.chunk_len = attn_split_chunk_len(Tk, num_splits);
    return dispatch_fwd<true>(D, q, k, v, prm, stream);
}

size_t attn_segments_workspace_bytes(int B, int H, int Tk, int D) {
    if (B <= 0 || H <= 0 || Tk <= 0 || D <= 0) return 0;
    const size_t kv = (static_cast<size_t>(B) * H * Tk * D * 2 + 255) / 256 * 256;
    return 2 * kv + (static_cast<size_t>(B) * sizeof(int32_t) + 255) / 256 * 256;
}

attn_status attn_prefix_fwd_segments(const void* q, const void* k, const void* v, const int32_t* seg_start,
                                     const int32_t* seg_len, int num_segments, void* workspace, void* out,
                                     float* lse, int B, int H, int Tq, int Tk, int D, float scale,
                                     cudaStream_t stream) {
    attn_status st = check_args(q, k, v, seg_start, out, B, H, Tq, Tk, D, scale);
    if (st != ATTN_OK) return st;
    if (!seg_len || (reinterpret_cast<uintptr_t>(seg_len) & 3u)) return ATTN_ERR_INVALID_ARG;
    if (num_segments < 1 || num_segments > attn::SEG_MAX_SEGMENTS) return ATTN_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return ATTN_ERR_INVALID_ARG;
    const long long n_rb = (static_cast<long long>(Tk) + attn::SEG_ROWS - 1) / attn::SEG_ROWS;
    const long long grid = n_rb * B * H;
    if (grid > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    if ((st = check_device()) != ATTN_OK) return st;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    const size_t kvb = (static_cast<size_t>(B) * H * Tk * D * 2 + 255) / 256 * 256;
    uint4* kg = reinterpret_cast<uint4*>(ws);
    uint4* vg = reinterpret_cast<uint4*>(ws + kvb);
    int32_t* kvl = reinterpret_cast<int32_t*>(ws + 2 * kvb);
    const size_t smem = (2 * static_cast<size_t>(num_segments) + 1) * sizeof(int);
    attn::gather_segments_kernel<<<static_cast<unsigned>(grid), attn::SEG_THREADS, smem, stream>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), kg, vg, seg_start, seg_len, num_segments, H,
        Tk, D * 2 / 16, static_cast<int>(n_rb), kvl);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    Params prm = base_params(kvl, B, H, Tq, Tk, D, scale);
    prm.out = static_cast<__nv_bfloat16*>(out);
    prm.lse = lse;
    return dispatch_fwd<false>(D, q, kg, vg, prm, stream);
}

attn_status attn_lse_combine_strided(const float* part_out, const float* part_lse, int num_splits, void* out,
                                     float* lse, int B, int H, int Tq, int D, const attn_strides* out_strides,
                                     cudaStream_t stream) {
    if (!part_out || !part_lse || !out) return ATTN_ERR_INVALID_ARG;
    Strides so;
    if (D <= 0 || !resolve_strides(out_strides, H, Tq, D, &so)) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(part_out) || !aligned16(out) || (reinterpret_cast<uintptr_t>(part_lse) & 3u) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return ATTN_ERR_INVALID_ARG;
    if (num_splits < 1 || num_splits > 1024 || B <= 0 || H <= 0 || Tq <= 0) return ATTN_ERR_INVALID_ARG;
    if (D != 32 && D != 64 && D != 128 && D != 256) return ATTN_ERR_UNSUPPORTED;
    attn_status st = check_device();
    if (st != ATTN_OK) return st;
    const long long rows = static_cast<long long>(B) * H * Tq;
    const long long blocks = (rows + 7) / 8;
    if (blocks > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
    const unsigned g = static_cast<unsigned>(blocks);
    switch (D) {
        case 32: attn::lse_combine_kernel<32><<<g, 256, 0, stream>>>(part_out, part_lse, num_splits, rows, H, Tq, o, so.b, so.h, so.t, lse); break;
        case 64: attn::lse_combine_kernel<64><<<g, 256, 0, stream>>>(part_out, part_lse, num_splits, rows, H, Tq, o, so.b, so.h, so.t, lse); break;
        case 128: attn::lse_combine_kernel<128><<<g, 256, 0, stream>>>(part_out, part_lse, num_splits, rows, H, Tq, o, so.b, so.h, so.t, lse); break;
        default: attn::lse_combine_kernel<256><<<g, 256, 0, stream>>>(part_out, part_lse, num_splits, rows, H, Tq, o, so.b, so.h, so.t, lse); break;
    }
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    return ATTN_OK;
}

attn_status attn_lse_combine(const float* part_out, const float* part_lse, int num_splits, void* out, float* lse,
                             int B, int H, int Tq, int D, cudaStream_t stream) {
    return attn_lse_combine_strided(part_out, part_lse, num_splits, out, lse, B, H, Tq, D, nullptr, stream);
}

attn_status attn_get_device_status(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    unsigned int flags = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&flags, attn::g_attn_status, sizeof flags) != cudaSuccess ||
        cudaMemcpyToSymbol(attn::g_attn_status, &zero, sizeof zero) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
    }
    if (flags & attn::STATUS_TIMEOUT) return ATTN_ERR_TIMEOUT;
    if (flags & attn::STATUS_KVLEN) return ATTN_ERR_KVLEN_RANGE;
    if (flags & attn::STATUS_LAYOUT) return ATTN_ERR_CUDA;
    return ATTN_OK;
}

void attn_set_wait_limit_ns(uint64_t ns) {
    g_wait_ns.store(ns < 1000000ull ? 1000000ull : ns, std::memory_order_relaxed);
}

void attn_set_debug_flags(unsigned flags) { g_debug.store(flags, std::memory_order_relaxed); }

const char* attn_status_string(attn_status s) {
    switch (s) {
        case ATTN_OK: return "ATTN_OK";
        case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
        case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
        case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
        case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
        case ATTN_ERR_KVLEN_RANGE: return "ATTN_ERR_KVLEN_RANGE";
    }
    return "ATTN_ERR_UNKNOWN";
}

int attn_version(void) { return 100; }

}  // extern "C"

// ------------------------------------------------------------------ no-allocation split-KV
// The partials of attn_prefix_fwd_splitkv_noalloc live here instead of in caller memory.
// In host code this name is only a host-side stand-in for the array: its device address
// comes from cudaGetSymbolAddress, looked up once per device with that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

namespace {

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// The driver's id of the current context (0 if it cannot be read).  A device reset or a
// context torn down and created again gets a new id, and may load the module -- and so
// the scratch array -- at a new address.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[64] = {};
unsigned long long g_noalloc_ctx[64] = {};

// Device address of the scratch array on the current device (nullptr on failure).  It is
// looked up with cudaGetSymbolAddress the first time a device is used, and again whenever
// that device's current context has changed since (a reset between calls).
void* noalloc_scratch_on_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return nullptr;
    }
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr || ctx == 0 || g_noalloc_ctx[dev] != ctx) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_noalloc_ptr[dev] = ptr;
        // read after the lookup, which creates the primary context if none existed yet
        g_noalloc_ctx[dev] = current_context_id();
    }
    return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" attn_status attn_prefix_fwd_splitkv_noalloc(const void* q, const void* k, const void* v,
                                                       const int32_t* kv_len, int num_splits, void* out, float* lse,
                                                       int B, int H, int Tq, int Tk, int D, float scale,
                                                       cudaStream_t stream) {
    attn_status st = check_args(q, k, v, kv_len, out, B, H, Tq, Tk, D, scale);
    if (st != ATTN_OK) return st;
    if (num_splits < 1 || num_splits > 1024) return ATTN_ERR_INVALID_ARG;
    const size_t need = attn_split_workspace_bytes(num_splits, B, H, Tq, D);
    if (need == 0 || need > static_cast<size_t>(ATTN_NOALLOC_SCRATCH_BYTES)) return ATTN_ERR_INVALID_ARG;
    if ((st = check_device()) != ATTN_OK) return st;
    unsigned char* scratch = static_cast<unsigned char*>(noalloc_scratch_on_current_device());
    if (scratch == nullptr) return ATTN_ERR_CUDA;
    float* part_out = reinterpret_cast<float*>(scratch);
    float* part_lse = reinterpret_cast<float*>(scratch + attn_split_lse_offset(num_splits, B, H, Tq, D));
    st = attn_prefix_fwd_split(q, k, v, kv_len, num_splits, part_out, part_lse, B, H, Tq, Tk, D, scale, stream);
    if (st != ATTN_OK) return st;
    return attn_lse_combine(part_out, part_lse, num_splits, out, lse, B, H, Tq, D, stream);
}
