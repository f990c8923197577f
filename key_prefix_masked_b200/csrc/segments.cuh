// Multi-range key mask: gather each batch element's key segments into a contiguous
// prefix, so the prefix kernels run unchanged on the gathered K/V.
//
// The gathered-shards K/V of "Add sequence-parallel multi-GPU inference ..." (section
// "Sequence-parallel inference": every device's context K/V is gathered with padded key
// slots) holds the valid keys of batch element b as one range per shard, not as one
// prefix.  Keys of the segments, in segment order, become rows [0, n_b) of the gathered
// buffers; n_b goes to kv_len.  Only rows inside a segment are read, so the padded
// slots between the shards never reach the attention.
//
// Segment s of element b is [seg_start[b*S+s], seg_start[b*S+s] + seg_len[b*S+s]),
// intersected with [0, Tk) (a negative length counts as 0); a key in two segments is
// gathered twice; the concatenation is cut after Tk keys.  A negative length, a
// non-empty segment reaching outside [0, Tk), or a cut raises the sticky
// kv-length-range flag.  Included by attn_prefix.cu inside namespace attn.

constexpr int SEG_ROWS = 64;            // gathered rows per CTA
constexpr int SEG_THREADS = 256;
constexpr int SEG_MAX_SEGMENTS = 4096;  // per batch element; shared memory 2(S+1) ints

// One CTA: gathered rows [rb * SEG_ROWS, +SEG_ROWS) of slice bh, where blockIdx.x =
// bh * n_rb + rb; K and V, one warp per row with 16-byte vectors.
__global__ void __launch_bounds__(SEG_THREADS) gather_segments_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, uint4* __restrict__ kg,
    uint4* __restrict__ vg, const int32_t* __restrict__ seg_start, const int32_t* __restrict__ seg_len,
    int S, int H, int Tk, int vec_per_row, int n_rb, int32_t* __restrict__ kv_len_out) {
    extern __shared__ int seg_smem[];
    int* s_lo = seg_smem;             // [S]     clamped segment start
    int* s_pre = seg_smem + S;        // [S + 1] exclusive prefix of clamped lengths
    __shared__ int s_warp_sum[SEG_THREADS / 32];
    const int bh = static_cast<int>(blockIdx.x / n_rb);
    const int rb = static_cast<int>(blockIdx.x % n_rb);
    const int b = bh / H;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;

    // ---- clamped lengths, then an exclusive scan (each thread a contiguous run of
    // segments).  Sums saturate at Tk + 1: a prefix past Tk is cut anyway, and
    // min(a + b, Tk + 1) is associative, so the saturated scan is exact below Tk.
    bool bad = false;
    const int per = (S + SEG_THREADS - 1) / SEG_THREADS;
    const int s0 = min(tid * per, S), s1 = min(s0 + per, S);
    const int cap = Tk + 1;
    int run = 0;
    for (int s = s0; s < s1; ++s) {
        const long long lo = seg_start[static_cast<long long>(b) * S + s];
        long long len = seg_len[static_cast<long long>(b) * S + s];
        if (len < 0) {
            bad = true;
            len = 0;
        }
        if (len > 0 && (lo < 0 || lo + len > Tk)) bad = true;
        const long long lo_c = lo < 0 ? 0 : (lo > Tk ? Tk : lo);
        const long long hi = lo + len;
        const long long hi_c = hi < 0 ? 0 : (hi > Tk ? Tk : hi);
        const int n = hi_c > lo_c ? static_cast<int>(hi_c - lo_c) : 0;
        s_lo[s] = static_cast<int>(lo_c);
        s_pre[s] = n;   // the length, until the scan below
        run = min(run + n, cap);
    }
    int incl = run;   // inclusive scan of the runs within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl = min(incl + t, cap);
    }
    int excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0;
    if (lane == 31) s_warp_sum[warp] = incl;
    __syncthreads();
    int acc = 0;
    for (int w = 0; w < warp; ++w) acc = min(acc + s_warp_sum[w], cap);
    acc = min(acc + excl, cap);   // exclusive prefix of this thread's first segment
    for (int s = s0; s < s1; ++s) {
        const int n = s_pre[s];
        s_pre[s] = min(acc, Tk);
        acc = min(acc + n, cap);
    }
    if (tid == SEG_THREADS - 1) {   // the runs of all other threads precede this one's
        s_pre[S] = min(acc, Tk);
        if (acc > Tk) bad = true;   // the concatenation was cut after Tk keys
    }
    if (__syncthreads_or(bad) && tid == 0) atomicOr(&g_attn_status, STATUS_KVLEN);
    const int total = s_pre[S];
    if (rb == 0 && (bh % H) == 0 && tid == 0) kv_len_out[b] = total;

    // ---- copy: gathered row r comes from key s_lo[s] + (r - s_pre[s]) of segment s,
    // the last segment with s_pre[s] <= r (empty segments share a prefix value and are
    // skipped by taking the last such s whose range is non-empty).
    const int r0 = rb * SEG_ROWS;
    const size_t slice = static_cast<size_t>(bh) * Tk;
    for (int r = r0 + warp; r < r0 + SEG_ROWS && r < total; r += SEG_THREADS / 32) {
        int lo = 0, hi = S - 1;   // largest s with s_pre[s] <= r and s_pre[s + 1] > r
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_pre[mid] <= r) lo = mid;
            else hi = mid - 1;
        }
        const int src = s_lo[lo] + (r - s_pre[lo]);
        const uint4* ks = k + (slice + src) * vec_per_row;
        const uint4* vs = v + (slice + src) * vec_per_row;
        uint4* kd = kg + (slice + r) * vec_per_row;
        uint4* vd = vg + (slice + r) * vec_per_row;
        for (int i = lane; i < vec_per_row; i += 32) {
            kd[i] = __ldg(ks + i);
            vd[i] = __ldg(vs + i);
        }
    }
}
