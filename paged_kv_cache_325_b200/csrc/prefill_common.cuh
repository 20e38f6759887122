// Block shape and roles, the register split, the sequence geometry and the planning kernel that writes the
// work-unit table of the prefill kernel (prefill.cu).  Included inside namespace pa { namespace { ... } } only.
#pragma once

constexpr int kM = 128;                // MMA rows per Q tile
constexpr int kN = 128;                // keys per K/V tile
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kFixWarp = 10;
constexpr int kQWarp = 11;
constexpr int kThreads = 384;          // 2 softmax warpgroups + K/V TMA warp + MMA warp + V-fix warp + Q TMA warp
constexpr int kVlast = 4;              // ring of last-V barriers: the K/V loads may run this many units ahead of
                                       // the V-fix warp
// Register split (setmaxnreg): a 384-thread block is launched with kRegsAtLaunch registers per thread (the
// most that ptxas gives it); the third warpgroup (TMA, MMA, V-fix, spare) drops to kRegsOther and the two
// softmax warpgroups, which hold a 128-column S row and a 128-column O row per thread, rise to kRegsSoftmax.
// The split must not ask for more than the block was launched with, or the increase waits forever: the
// host checks the compiled register count before every first launch.
constexpr uint32_t kRegsAtLaunch = 168;
constexpr uint32_t kRegsOther = 136;
constexpr uint32_t kRegsSoftmax = 184;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther <= kThreads * kRegsAtLaunch, "register split");
constexpr int kRowBytes = 128;         // one 64-element bf16 swizzle row
constexpr int kSlab = kM * kRowBytes;  // 128 rows x 128 B = 16 KB
constexpr int kUnitQueue = 4;          // unit ids handed from the TMA warp to the other roles
// Ring of "last V tile fixed" barriers, one entry per unit in turn.  The V-fix warp may run ahead of the MMA
// thread, but by fewer than kFixRing units: it fixes unit m only after the K/V warp pushed m to the unit queue,
// which needs every consumer, the MMA thread included, to have popped unit m - kUnitQueue; the MMA thread pops
// a unit only after finishing the one before, so it has waited for the fix of unit m - kUnitQueue - 1 and
// earlier.  Entry m % kFixRing is therefore never two phases ahead of its waiter.
constexpr int kFixRing = 2 * kUnitQueue;
static_assert(kFixRing > kUnitQueue + 1, "fix ring deeper than the unit queue's lead");
constexpr int kPlanThreads = 1024;

// Geometry of one sequence; false when its cu_seqlens are inconsistent.
__device__ __forceinline__ bool seq_geometry(const PrefillArgs &a, int s, int &q0, int &n_new, int &n_k) {
    if (!a.cu_q) {                    // one sequence given by scalars
        q0 = 0;
        n_new = a.single_n_new;
        n_k = a.single_n_k;
        return s == 0 && n_new >= 0 && n_k >= 1 && n_new <= a.total_q && n_new <= a.max_seqlen_q &&
               n_k <= a.max_seqlen_k && (int64_t)n_k <= (int64_t)a.bt_stride * a.block_size;
    }
    q0 = a.cu_q[s];
    const int q1 = a.cu_q[s + 1];
    const int k0 = a.cu_k[s], k1 = a.cu_k[s + 1];
    n_new = q1 - q0;
    n_k = k1 - k0;
    return !(n_new < 0 || n_k < n_new || q0 < 0 || k0 < 0 || q1 > a.total_q || n_new > a.max_seqlen_q ||
             n_k > a.max_seqlen_k || (int64_t)n_k > (int64_t)a.bt_stride * a.block_size);
}

// Work-unit table written by prefill_plan_kernel into the workspace (int32 words):
//   w[0] hand-out counter, w[1] number of units, w[2] R (ranks)
//   prefix[R + 1] at word 16: units in ranks < r
//   order[batch]: sequences, longest first
//   geo[batch] (int4, 16-byte aligned): q0, n_new, n_k, valid of every sequence
//   units[R * batch * Hkv] (int4): s, kv head, rank of every unit, in hand-out order
// Unit u has rank r = the r-th group of Q tiles (two tiles: `tokens_per_unit` new tokens) counted from the end
// of its sequence; ranks come in
// increasing order and, within a rank, sequences longest first, so the list runs from the most to the
// least expensive unit and a greedy hand-out balances the CTAs.
struct PlanLayout {
    int32_t prefix, order, geo, units;   // word offsets
};

__host__ __device__ __forceinline__ PlanLayout plan_layout(int32_t R, int32_t batch) {
    PlanLayout l;
    l.prefix = 16;
    l.order = l.prefix + R + 1;
    l.geo = (l.order + batch + 3) & ~3;
    l.units = l.geo + 4 * batch;
    return l;
}

// One CTA: validate every sequence, sort the sequences by their number of units (longest first),
// count the units of every rank, write the prefix sums and zero the hand-out counter.
__global__ void __launch_bounds__(kPlanThreads)
    prefill_plan_kernel(const PrefillArgs a, int32_t R, int32_t tokens_per_unit) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // the main kernel may start its prologue
    extern __shared__ int32_t plan_smem[];
    int32_t *np = plan_smem;                  // [batch] pairs per sequence
    int32_t *nps = plan_smem + a.batch;       // [batch] pairs, sorted descending
    __shared__ int32_t warp_tot[32];
    int32_t *w = static_cast<int32_t *>(a.workspace);
    const PlanLayout lay = plan_layout(R, a.batch);
    int32_t *prefix = w + lay.prefix;
    int32_t *order = w + lay.order;
    int4 *geo = reinterpret_cast<int4 *>(w + lay.geo);
    int4 *units = reinterpret_cast<int4 *>(w + lay.units);
    const int tid = threadIdx.x;
    for (int s = tid; s < a.batch; s += kPlanThreads) {
        int q0, n_new, n_k;
        if (seq_geometry(a, s, q0, n_new, n_k)) {
            // a mixed batch's one-token sequences are the decode kernel's work
            np[s] = (a.skip_single && n_new == 1) ? 0 : min(R, (n_new + tokens_per_unit - 1) / tokens_per_unit);
            geo[s] = make_int4(q0, n_new, n_k, 1);
        } else {
            np[s] = 0;
            geo[s] = make_int4(0, 0, 0, 0);
            report(a.dev_error, PA_DEVERR_SEQLENS);
        }
    }
    __syncthreads();
    for (int s = tid; s < a.batch; s += kPlanThreads) {
        const int v = np[s];
        int rank = 0;
        for (int t = 0; t < a.batch; ++t) rank += (np[t] > v) || (np[t] == v && t < s);
        order[rank] = s;
        nps[rank] = v;
    }
    __syncthreads();
    // units of rank r = Hkv * #{s : np[s] > r}; nps is descending, so count by binary search
    const int chunk = (R + kPlanThreads - 1) / kPlanThreads;
    const int r0 = min(R, tid * chunk), r1 = min(R, r0 + chunk);
    int32_t local = 0;
    for (int r = r0; r < r1; ++r) {
        int lo = 0, hi = a.batch;                 // first index with nps <= r
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (nps[mid] > r) lo = mid + 1; else hi = mid;
        }
        local += lo * a.num_kv_heads * a.nchunks;
    }
    // exclusive block scan of `local`
    const int lane = tid & 31, wid = tid >> 5;
    int32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int32_t t = warp_tot[lane], ti = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, ti, o);
            if (lane >= o) ti += y;
        }
        warp_tot[lane] = ti - t;                  // exclusive prefix of the warp totals
    }
    __syncthreads();
    int32_t run = warp_tot[wid] + incl - local;
    for (int r = r0; r < r1; ++r) {
        prefix[r] = run;
        int lo = 0, hi = a.batch;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (nps[mid] > r) lo = mid + 1; else hi = mid;
        }
        run += lo * a.num_kv_heads * a.nchunks;
    }
    if (r1 == R && r0 < R) prefix[R] = run;
    if (R == 0 && tid == 0) prefix[0] = 0;
    __syncthreads();                              // prefix and order are visible to the whole CTA
    const int total = prefix[R];
    for (int u = tid; u < total; u += kPlanThreads) {
        int lo = 0, hi = R;                       // prefix[lo] <= u < prefix[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (prefix[mid] <= u) lo = mid; else hi = mid;
        }
        const int i = u - prefix[lo];
        const int per_seq = a.num_kv_heads * a.nchunks;
        units[u] = make_int4(order[i / per_seq], (i % per_seq) / a.nchunks, lo, i % a.nchunks);
    }
    if (tid == 0) {
        w[0] = 0;                                 // hand-out counter
        w[1] = total;
        w[2] = R;
    }
}

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}
