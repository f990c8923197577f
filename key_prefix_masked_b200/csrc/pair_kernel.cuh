// pair_kernel.cuh -- forward on a CTA pair (cta_group::2) for head dims 128 and 256.
// Included by attn_prefix.cu inside namespace attn, after the single-CTA kernel's helpers.
//
// A cluster of two CTAs shares one 256-row query tile: each CTA holds its own 128 query
// rows (Q in its shared memory, S / P / O in its TMEM lanes) and HALF of every key and
// value tile -- keys [64r, 64r + 64) of K, value columns [r*D/2, (r+1)*D/2) of V for
// CTA rank r.  The leader CTA's MMA warp issues M = 256 tcgen05 MMAs that read A from
// each CTA and B split across both, so each CTA streams half of every K/V tile (64 KB at
// D=256, 32 KB at D=128) and one instruction covers 256 rows: at D=256 the five 32 KB ring slots hold 2.5 tiles of look-ahead, at D=128 twelve
// 16 KB slots hold 6.  MMA order: S_0, S_1, then PV_j, S_{j+2} per tile j; P_j is stored
// over S_j, and S_{j+2} overwrites it only after PV_j has read it (one thread's MMAs run
// in issue order).
//
// Roles at D=256 (224 threads per CTA): warps 0-3 softmax + epilogue (both CTAs); warp 4
// copy producer (both CTAs, into their own memory, completing on the leader's barriers);
// warp 5 TMEM allocation (both) and MMA issue (leader); warp 6 wait relay (leader).
// At D=128 the kernel runs in two-group mode (352 threads: softmax warps 0-7, then the
// same three roles): warpgroup w takes the key tiles j = w (mod 2) with its own running
// max, row sum and TMEM O accumulator O_w (S_0, S_1, O_0, O_1 fill the 512 columns), so
// one group's softmax overlaps the other's P -> PV -> S round trip; the two warps that
// share a sub-partition run their exponentials whenever their tiles are ready (turns in
// tile order cost 5 to 8 % once the MMA warp stopped spinning); the two partial results
// are merged exactly at the end by the log-sum-exp rule of split-KV ("Sequence-parallel inference"
// of "Add sequence-parallel multi-GPU inference ... and a cuDNN flash attention option").
// S_j is issued after PV_{j-2}, the last PV into O_{j&1} before tile j, so "S_j ready"
// already means that accumulator is quiescent and the group rescales it without waiting.
//
// Each softmax warp of either CTA announces P with one arrival on the leader's P
// barrier (the remote mbarrier arrive with default semantics -- release at CTA scope --
// which is the cross-CTA handshake the pair pipelines are built on; a cluster-scope
// release costs ~450-1100 cycles and made this handshake the critical path).  The relay
// publishes the copies' arrivals; the MMA warp waits for "P_j stored in both CTAs" itself.
//
// The last, partial key tile of a range is read as the window [k_end - 128, k_end):
// every row copied is a valid key (or a zero-filled row at a negative coordinate), and
// the columns that belong to earlier tiles or ranges are masked by selection, so key
// padding is never read.

constexpr int PAIR_MAX_SLOTS = 12;

template <int D_>
struct PairCfg {
    static constexpr int D = D_;
    static constexpr int ROWS = 128;                 // query rows per CTA (TMEM lanes)
    static constexpr int NBLK = D / 64;              // 64-column (128-byte) blocks per row
    static constexpr int Q_BYTES = ROWS * D * 2;     // 64 KB at D=256
    static constexpr int KH = BN / 2;                // keys of a K tile held by one CTA
    static constexpr int KBLK_BYTES = KH * 128;      // one 64-column block of them: 8 KB
    static constexpr int VBLK_BYTES = BN * 128;      // one 64-column block of V: 16 KB
    static constexpr int SLOT = NBLK * KBLK_BYTES;   // one CTA's half of a K or V tile
    // Two-group mode (head dim 128): two softmax warpgroups on alternate key tiles, each
    // with its own O accumulator; S_0, S_1, O_0, O_1 fill the 512 TMEM columns.
    static constexpr bool DUAL = O_COL + 2 * D <= TMEM_COLS;
    static constexpr int SM_WARPS = DUAL ? 8 : 4;    // softmax warps
    static constexpr int WARP_PROD = SM_WARPS;       // copy producer (both CTAs)
    static constexpr int WARP_MMA = SM_WARPS + 1;    // TMEM owner (both), MMA issuer (leader)
    static constexpr int WARP_RELAY = SM_WARPS + 2;  // wait relay (leader)
    static constexpr int THREADS = 32 * (SM_WARPS + 3);
    static constexpr int CTRL = 1024;
    static constexpr int XCH_BYTES = DUAL ? 2 * 2 * ROWS * 4 : 0;   // per-group (max, sum) exchange
    static constexpr int NSLOTS_FIT = (SMEM_LIMIT - Q_BYTES - CTRL - XCH_BYTES) / SLOT;
    static constexpr int NSLOTS = NSLOTS_FIT < PAIR_MAX_SLOTS ? NSLOTS_FIT : PAIR_MAX_SLOTS;
    static constexpr int SMEM_BYTES = Q_BYTES + NSLOTS * SLOT + CTRL + XCH_BYTES;
    // Who waits for "P_j stored": the MMA warp itself, with a suspending try_wait, which
    // takes the relay's wake-up off the P -> PV handshake (measured, same-box A/B against
    // the relay doing that wait: +6.5 % on icl and +6.1 % on ragged at D=256, +2 to +4 %
    // at D=128; a spinning test_wait from one thread had cost 1.5 % at D=256).
    static constexpr bool MMA_WAITS_P = true;
    static_assert(D == 128 || D == 256, "pair head dims");
    static_assert(NSLOTS >= 4, "pair ring depth");
    static_assert(SMEM_BYTES <= SMEM_LIMIT && 2 * SMEM_BYTES > SMEM_LIMIT, "one CTA per SM, within budget");
    static_assert((NBLK / 2) * VBLK_BYTES == SLOT, "a V half fills a slot like a K half");
    static_assert(O_COL + D <= TMEM_COLS, "pair TMEM budget");
};

enum : int {
    PB_Q = 0,
    PB_FULL = 1,     // [PAIR_MAX_SLOTS] slot filled by both CTAs' copies (leader)
    PB_EMPTY = 13,   // [PAIR_MAX_SLOTS] slot consumed (multicast commit, both CTAs)
    PB_S = 25,       // [2] S_j ready (multicast commit, both CTAs)
    PB_OLAST = 27,   // PV_{n-1} complete (multicast commit, both CTAs; completes once)
    PB_DRAIN = 28,   // leader only
    PB_P = 29,       // [2] P_j stored by both CTAs' softmax warps (leader; 8 warp arrivals)
    PB_OPREV = 31,   // PV_{n-2} complete (multicast commit, both CTAs; completes once)
    PB_NUM = 32
};
static_assert(PB_EMPTY == PB_FULL + PAIR_MAX_SLOTS && PB_S == PB_EMPTY + PAIR_MAX_SLOTS, "pair barrier map");

template <int D, bool SPLIT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<D>::THREADS, 1)
    attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const Params p) {
    using C = PairCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    // Swizzled tiles need 1024-byte alignment; both CTAs see the same layout, so both
    // return here together (no cluster barrier has been reached yet).
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicOr(&g_attn_status, STATUS_LAYOUT);
        return;
    }
    uint8_t* sQ = smem;
    uint8_t* sKV = smem + C::Q_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + C::NSLOTS * C::SLOT);
    uint32_t* words = reinterpret_cast<uint32_t*>(bars + PB_NUM);   // tmem, abort, relay seq, fused-combine flag
    volatile int* abort_flag = reinterpret_cast<volatile int*>(words + 1);
    const uint32_t bar0 = smem_u32(bars);
    const uint32_t sQ_addr = smem_u32(sQ);
    const uint32_t sKV_addr = smem_u32(sKV);
    const uint32_t seq_addr = smem_u32(words + 2);
#define PBAR(i) (bar0 + 8u * static_cast<uint32_t>(i))

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    // ---- work unit of the pair: 256-row query tile fastest, then split chunk, then (b, h)
    int unit = static_cast<int>(blockIdx.x >> 1);
    const int ptile = unit % p.n_qtiles;
    unit /= p.n_qtiles;
    const int split = SPLIT ? unit % p.num_splits : 0;
    const int bh = SPLIT ? unit / p.num_splits : unit;
    const int b = bh / p.H;
    const int h = bh - b * p.H;
    const int q0 = ptile * (2 * C::ROWS) + static_cast<int>(rank) * C::ROWS;

    int kv = __ldg(p.kv_len + b);
    if (kv < 0 || kv > p.Tk) {
        if (tid == 0 && leader) atomicOr(&g_attn_status, STATUS_KVLEN);
        kv = kv < 0 ? 0 : p.Tk;
    }
    const int k_begin = SPLIT ? split * p.chunk_len : 0;
    const int k_end = SPLIT ? min(kv, k_begin + p.chunk_len) : kv;
    const int n_tiles = (k_end > k_begin) ? (k_end - k_begin + BN - 1) / BN : 0;
    // leading columns of the last tile that belong to earlier tiles (0 when it is full)
    const int last_lo = n_tiles > 0 ? n_tiles * BN - (k_end - k_begin) : 0;
    auto tile_key0 = [&](int j) { return (j == n_tiles - 1 && last_lo > 0) ? k_end - BN : k_begin + j * BN; };

    if (tid == 0) {
        mbar_init(PBAR(PB_Q), 1);
        for (int s = 0; s < C::NSLOTS; ++s) {
            mbar_init(PBAR(PB_FULL + s), 1);
            mbar_init(PBAR(PB_EMPTY + s), 1);
        }
        mbar_init(PBAR(PB_S + 0), 1);
        mbar_init(PBAR(PB_S + 1), 1);
        mbar_init(PBAR(PB_OLAST), 1);
        mbar_init(PBAR(PB_OPREV), 1);
        mbar_init(PBAR(PB_DRAIN), 1);
        mbar_init(PBAR(PB_P + 0), 8);
        mbar_init(PBAR(PB_P + 1), 8);
        words[1] = 0u;
        words[2] = 0u;
        fence_mbar_init();
    }
    if (warp == C::WARP_MMA) {
        tmem_alloc_pair(smem_u32(words), TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = words[0];
    const unsigned long long wlim = p.wait_ns;

    if (warp == C::WARP_PROD) {
        // ================================================================ producer (both CTAs)
        if (lane == 0 && n_tiles > 0) {
            tma_prefetch_map(&tm_q);
            tma_prefetch_map(&tm_k);
            tma_prefetch_map(&tm_v);
            if (leader) mbar_arrive_expect_tx(PBAR(PB_Q), 2 * C::Q_BYTES);
            const uint32_t lq = mapa_shared(PBAR(PB_Q), 0);
            // Q is read once: evict it first.  Every pair of the head streams the head's K/V,
            // so half of its lines are kept in L2 ahead of Q and of the output stream.  Half,
            // not all: where the resident clusters span two heads whose K/V together exceed
            // L2 (2 x 102 MB at 100000 keys, D=256), protected lines of both heads would
            // evict one another; the protected halves of two heads fit.
            const uint64_t pol_q = l2_policy_evict_first();
            const uint64_t pol_kv = l2_policy_evict_last_half();
#pragma unroll
            for (int blk = 0; blk < C::NBLK; ++blk)
                tma_load_4d_pair_hint(sQ_addr + blk * (C::ROWS * 128), &tm_q, blk * 64, q0, h, b, lq, pol_q);
            int slot = 0;
            uint32_t phase = 0;
            bool ok = true;
            auto item = [&](bool is_k, int j) {
                if (!ok) return;
                ok = wait_bar(PBAR(PB_EMPTY + slot), phase ^ 1u, abort_flag, wlim);
                if (!ok) return;
                if (leader) mbar_arrive_expect_tx(PBAR(PB_FULL + slot), 2 * C::SLOT);
                const uint32_t lfull = mapa_shared(PBAR(PB_FULL + slot), 0);
                const uint32_t dst = sKV_addr + slot * C::SLOT;
                const int key0 = tile_key0(j);
                if (is_k) {
                    const bool drop = (p.debug & ATTN_DEBUG_DROP_COPY) && leader && j == 0;
#pragma unroll
                    for (int c = 0; c < C::NBLK; ++c)
                        if (!(drop && c == 0))
                            tma_load_4d_pair_hint(dst + c * C::KBLK_BYTES, &tm_k, c * 64,
                                                  key0 + static_cast<int>(rank) * C::KH, h, b, lfull, pol_kv);
                } else {
#pragma unroll
                    for (int c = 0; c < C::NBLK / 2; ++c)
                        tma_load_4d_pair_hint(dst + c * C::VBLK_BYTES, &tm_v, static_cast<int>(rank) * (D / 2) + c * 64,
                                              key0, h, b, lfull, pol_kv);
                }
                if (++slot == C::NSLOTS) {
                    slot = 0;
                    phase ^= 1u;
                }
            };
            for (int i = 0; i < 2 && i < n_tiles; ++i) item(true, i);
#pragma unroll 1
            for (int j = 0; j < n_tiles && ok; ++j) {
                item(false, j);
                if (j + 2 < n_tiles) item(true, j + 2);
            }
            if (!ok) {
                // Copies already issued complete on the leader's barriers; give them time to
                // land before this CTA's memory can be reused.
                const uint64_t t0 = global_timer_ns();
                while (global_timer_ns() - t0 < 2000000ull) {
                }
            }
        }
        __syncwarp();
    } else if (warp == C::WARP_RELAY) {
        // ================================================================ wait relay (leader)
        // Waits on Q and, in the MMA warp's consumption order, on K_0, K_1, then per tile
        // V_j and K_{j+2}; publishes the count of completed events with a release store.
        if (leader && lane == 0 && n_tiles > 0) {
            uint32_t seq = 0;
            bool ok = wait_bar(PBAR(PB_Q), 0, abort_flag, wlim);
            if (ok) st_release_smem(seq_addr, ++seq);
            int slot = 0;
            uint32_t phase = 0;
            auto item = [&]() {
                ok = ok && wait_bar(PBAR(PB_FULL + slot), phase, abort_flag, wlim);
                if (++slot == C::NSLOTS) {
                    slot = 0;
                    phase ^= 1u;
                }
            };
            auto publish = [&]() {
                if (ok) st_release_smem(seq_addr, ++seq);
            };
            for (int i = 0; i < 2 && i < n_tiles; ++i) {
                item();  // K_i
                publish();
            }
#pragma unroll 1
            for (int j = 0; j < n_tiles && ok; ++j) {
                item();  // V_j
                if constexpr (!C::MMA_WAITS_P)
                    ok = ok && wait_bar(PBAR(PB_P + (j & 1)), (j >> 1) & 1, abort_flag, wlim);
                publish();
                if (j + 2 < n_tiles) {
                    item();  // K_{j+2}
                    publish();
                }
            }
        }
        __syncwarp();
    } else if (warp == C::WARP_MMA) {
        // ================================================================ MMA issuer (leader)
        // The whole warp runs the issuing code converged and its elected lane issues every
        // MMA and commit, so the descriptors stay warp-uniform (measured on B200: 68 cycles
        // per MMA issued this way against 83 from one thread of a divergent branch; at
        // D=256 an S MMA executes in 64, so the issue rate bounds the S phase).  Every wait
        // decision is lane 0's, broadcast, so the warp stays converged.
        if (leader && n_tiles > 0) {
            constexpr uint32_t IDESC_S = make_idesc_bf16(2 * C::ROWS, BN, false);
            constexpr uint32_t IDESC_PV = make_idesc_bf16(2 * C::ROWS, D, true);
            const uint64_t q_desc0 = make_smem_desc(sQ_addr, 16, 1024, 2);
            const uint64_t k_desc0 = make_smem_desc(sKV_addr, 16, 1024, 2);
            const uint64_t v_desc0 = make_smem_desc(sKV_addr, C::VBLK_BYTES, 1024, 2);
            int slot = 0;
            uint32_t consumed = 0;
            auto uniform = [&](bool v) { return __shfl_sync(0xffffffffu, v ? 1 : 0, 0) != 0; };
            // lane 0 reads the relay's count and broadcasts it (one shared-memory load per poll)
            auto poll_word = [&](uint32_t addr) -> uint32_t {
                uint32_t v = 0;
                if (lane == 0) v = ld_acquire_cluster_smem(addr);
                return __shfl_sync(0xffffffffu, v, 0);
            };
            // A failed poll backs off (nanosleep) before the next one: this warp shares its
            // sub-partition with a softmax warp, and a spinning poll takes its issue slots.
            auto poll_ge = [&](uint32_t addr, uint32_t need) -> bool {
                bool ok_p = true;
                if (poll_word(addr) < need) {
                    const uint64_t t0 = global_timer_ns();
                    while (true) {
                        __nanosleep(32);
                        if (poll_word(addr) >= need) break;
                        if (*abort_flag) {
                            ok_p = false;
                            break;
                        }
                        if (global_timer_ns() - t0 > wlim) {
                            if (lane == 0) {
                                *abort_flag = 1;
                                atomicOr(&g_attn_status, STATUS_TIMEOUT);
                            }
                            ok_p = false;
                            break;
                        }
                    }
                }
                return uniform(ok_p);
            };
            auto slot_desc = [&](uint64_t d0) { return d0 + static_cast<uint64_t>(slot) * (C::SLOT >> 4); };
            auto next_slot = [&]() { slot = (slot + 1 == C::NSLOTS) ? 0 : slot + 1; };
            bool ok = poll_ge(seq_addr, ++consumed);   // both Q tiles landed
            auto issue_s = [&](int j) {
                ok = poll_ge(seq_addr, ++consumed);     // K_j halves landed in both CTAs
                if (!ok) return;
                tc_fence_after();
                const uint32_t d_tmem = tmem + static_cast<uint32_t>(j & 1) * BN;
                const uint64_t kd = slot_desc(k_desc0);
#pragma unroll
                for (int t = 0; t < D / 16; ++t) {
                    const int c = t >> 2, kk = t & 3;
                    mma_ss_pair_elect(d_tmem, q_desc0 + static_cast<uint64_t>(((c * C::ROWS * 128) >> 4) + kk * 2),
                                      kd + static_cast<uint64_t>(((c * C::KBLK_BYTES) >> 4) + kk * 2), IDESC_S, t != 0);
                }
                tc_commit_pair_elect(PBAR(PB_EMPTY + slot), 0x3);
                tc_commit_pair_elect(PBAR(PB_S + (j & 1)), 0x3);
                next_slot();
            };
            auto issue_pv = [&](int j) {
                ok = poll_ge(seq_addr, ++consumed);   // V_j halves landed
                if (!ok) return;
                if constexpr (C::MMA_WAITS_P) {
                    // P_j stored in both CTAs: waited here with try_wait, which suspends the
                    // warp (no issue slots taken from the softmax warp beside it)
                    const uint32_t pb = PBAR(PB_P + (j & 1));
                    const uint32_t par = (j >> 1) & 1;
                    if (!uniform(mbar_try_wait(pb, par))) {
                        const uint64_t t0 = global_timer_ns();
                        while (true) {
                            if (uniform(mbar_try_wait(pb, par))) break;
                            if (uniform(*abort_flag != 0)) {
                                ok = false;
                                return;
                            }
                            if (uniform(global_timer_ns() - t0 > wlim)) {
                                if (lane == 0) {
                                    *abort_flag = 1;
                                    atomicOr(&g_attn_status, STATUS_TIMEOUT);
                                }
                                ok = false;
                                return;
                            }
                        }
                    }
                }
                tc_fence_after();
                // PV_j reads P_j (over S_j); two-group mode: it adds into O_{j&1}, and
                // each accumulator starts fresh
                const uint32_t p_tmem = tmem + static_cast<uint32_t>(j & 1) * BN;
                const uint32_t o_tmem = tmem + O_COL + (C::DUAL ? static_cast<uint32_t>((j & 1) * D) : 0u);
                const uint32_t acc0 = (j < (C::DUAL ? 2 : 1)) ? 0u : 1u;
                const uint64_t vd = slot_desc(v_desc0);
#pragma unroll
                for (int kb = 0; kb < BN / 16; ++kb)
                    mma_ts_pair_elect(o_tmem, p_tmem + static_cast<uint32_t>(kb) * 8u,
                                      vd + static_cast<uint64_t>((kb * 16 * 128) >> 4), IDESC_PV, kb == 0 ? acc0 : 1u);
                tc_commit_pair_elect(PBAR(PB_EMPTY + slot), 0x3);
                // Each O barrier completes exactly once, so a parity-0 wait on it cannot
                // be confused by a later phase.
                if (!C::DUAL && j == n_tiles - 2) tc_commit_pair_elect(PBAR(PB_OPREV), 0x3);
                if (j == n_tiles - 1) tc_commit_pair_elect(PBAR(PB_OLAST), 0x3);
                next_slot();
            };
            for (int i = 0; i < 2 && i < n_tiles && ok; ++i) issue_s(i);
#pragma unroll 1
            for (int j = 0; j < n_tiles && ok; ++j) {
                issue_pv(j);
                if (ok && j + 2 < n_tiles) issue_s(j + 2);
            }
            tc_commit_pair_elect(PBAR(PB_DRAIN), 0x1);
            __syncwarp();
            wait_bar_drain(PBAR(PB_DRAIN), 0, wlim);
        }
        __syncwarp();
    } else if (warp < C::SM_WARPS) {
        // ================================================================ softmax (both CTAs)
        // Thread t of warpgroup w owns query row q0 + t % 128 (TMEM lane t % 128).  Two-group
        // mode: group w takes the key tiles j = w (mod 2) with its own running max, row sum
        // and O accumulator O_w, and the two partial results are merged exactly at the end
        // (the log-sum-exp rule of split-KV); otherwise group 0 takes every tile.
        constexpr bool DUAL = C::DUAL;
        const int wg = warp >> 2;
        const int r = tid & 127;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t o_col = O_COL + (DUAL ? static_cast<uint32_t>(wg * D) : 0u);
        const float sl2 = p.scale_log2;
        const bool pos_scale = sl2 > 0.0f;
        float m_ref = -INFINITY;
        float l_sum = 0.0f;
        bool ok = true;
        int seen = 0;   // tiles this group has processed
#pragma unroll 1
        for (int j = DUAL ? wg : 0; j < n_tiles; j += DUAL ? 2 : 1) {
            // Two-group mode: S_j was issued after PV_{j-2}, the last PV into O_w before
            // this tile, and its commit completes after every earlier MMA: from here on O_w
            // is quiescent until PV_j, which needs this tile's P.
            ok = __all_sync(0xffffffffu, wait_bar(PBAR(PB_S + (j & 1)), (j >> 1) & 1, abort_flag, wlim));
            if (!ok) break;
            tc_fence_after();
            const uint32_t s_addr = tmem + lane_base + static_cast<uint32_t>(j & 1) * BN;
            uint32_t raw[BN];
            tmem_ld128_wait(s_addr, raw);
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
#pragma unroll
                for (int c = 0; c < BN; ++c) x[c] = (c >= lo) ? x[c] * sl2 : -INFINITY;
            }
            const float mx = row_max(x) * (pos_scale ? sl2 : 1.0f);   // three-input maxima
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
            // p = 2^(x * mul - m): the scale-and-shift and the row sum in packed pairs
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
                tmem_st16(s_addr + cc * 16, pk);
            }
            const float tile_sum = ((sp[0].x + sp[1].x) + (sp[2].x + sp[3].x)) + ((sp[0].y + sp[1].y) + (sp[2].y + sp[3].y));
            l_sum = l_sum * factor + tile_sum;
            if (rescale) {
                if constexpr (!DUAL) {
                    // PV_{j-1} is complete once S_{j+1} (issued after it) is; for the last
                    // tile the leader announces PV_{n-2} on its own barrier.
                    const bool w = (j + 1 < n_tiles)
                                       ? wait_bar(PBAR(PB_S + ((j + 1) & 1)), ((j + 1) >> 1) & 1, abort_flag, wlim)
                                       : wait_bar(PBAR(PB_OPREV), 0, abort_flag, wlim);
                    ok = __all_sync(0xffffffffu, w);
                    if (!ok) break;
                    tc_fence_after();
                }
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
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(mapa_shared(PBAR(PB_P + (j & 1)), 0));
            ++seen;
        }
        // ---- epilogue
        if (ok && n_tiles > 0) {
            // PV_{n-1}'s commit tracks every earlier MMA of the leader's thread as well
            const bool w = wait_bar(PBAR(PB_OLAST), 0, abort_flag, wlim);
            ok = __all_sync(0xffffffffu, w);
            tc_fence_after();
        }
        // Two-group mode: m = max_w m_w, f_w = 2^(m_w - m), l = sum_w l_w f_w,
        // O = sum_w O_w f_w / l (a group with no tile has l_w = 0 and weight 0).
        float f_own = 1.0f, f_other = 0.0f, m_row = m_ref, l_row = l_sum;
        bool own_has = n_tiles > 0, other_has = false;
        if constexpr (DUAL) {
            float* xch = reinterpret_cast<float*>(sKV + C::NSLOTS * C::SLOT + C::CTRL);   // [2][max, sum][128]
            xch[(wg * 2 + 0) * 128 + r] = m_ref;
            xch[(wg * 2 + 1) * 128 + r] = l_sum;
            named_barrier_sync(XCH_ID, 32 * C::SM_WARPS);
            const float m_o = xch[((wg ^ 1) * 2 + 0) * 128 + r];
            const float l_o = xch[((wg ^ 1) * 2 + 1) * 128 + r];
            own_has = l_sum > 0.0f;
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
        const uint32_t o_col_other = O_COL + static_cast<uint32_t>((wg ^ 1) * D);
        // two-group mode: group w writes the 32-column chunks oc = w (mod 2)
#pragma unroll 1
        for (int oc = DUAL ? wg : 0; oc < D / 32; oc += DUAL ? 2 : 1) {
            uint32_t o[32];
            if (have && own_has) {
                tmem_ld32_wait(tmem + lane_base + o_col + oc * 32, o);
                if constexpr (DUAL) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f_own);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = 0u;
            }
            if (DUAL && have && other_has) {
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
                    __stcs(reinterpret_cast<uint4*>(dst + e), v4);   // streaming: out is not read again
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

    // Neither CTA may release its TMEM or leave while the pair's MMAs, commits or copies
    // may still touch the other one.
    tc_fence_before();
    cluster_sync();
    if (warp == C::WARP_MMA) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
    if constexpr (SPLIT) {
        if (p.counters != nullptr)
            fused_combine_tail<D>(p, bh, q0, tid, C::THREADS, reinterpret_cast<volatile int*>(words + 3));
    }
#undef PBAR
}
