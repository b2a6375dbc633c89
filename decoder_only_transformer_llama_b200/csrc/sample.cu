// Next-token selection (Admin Guide §6.3 and §8.5; source tour, sample_top_p).
//
// Greedy: argmax over the vocabulary, lowest id on ties.
//
// Top-p: p = softmax(l / T); tokens ordered by p descending, ties by id
// ascending; token k is kept iff the mass before it is <= top_p; the draw is
// the first kept token whose cumulative mass exceeds u * (kept mass).
// The reference sorts the whole vocabulary; here one CTA per row finds the
// two tokens that matter (the last kept one and the drawn one) without a
// sort, by a most-significant-digit radix select over a 64-bit order key
//     key = ordered_bits(logit) << 32 | ~id      (descending key = sampling order)
// using histograms of probability mass: the first-digit histogram of the whole
// row (which also gives the total mass) serves both selects, and once a chosen
// digit prefix holds at most kListCap keys they are copied into shared memory
// and the remaining passes read only them.  Masses are e_i = exp((l_i - l_max)/T)
// evaluated in fp64 and held as 64-bit fixed point (2^-46 resolution), so
// every prefix sum is an exact integer and the result does not depend on the
// summation order.
#include "common.cuh"
#include "model.h"

namespace llb {

namespace {
constexpr int kSampleThreads = 1024;
constexpr int kWarps = kSampleThreads / 32;
constexpr double kFixScale = 70368744177664.0;    // 2^46: V * 2^46 < 2^64 for V <= 262144
}

__device__ __forceinline__ uint32_t ordered_bits(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint64_t sort_key(float l, int id) {
    return (static_cast<uint64_t>(ordered_bits(l)) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(id));
}

// ---------------------------------------------------------------- argmax
__global__ void __launch_bounds__(kSampleThreads)
argmax_kernel(const float* __restrict__ logits, int V, int32_t* out, int32_t* tokens_adv, int32_t* pos_adv,
              unsigned long long* tl) {
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x;
    const float* row = logits + static_cast<long long>(b) * V;
    float best = -INFINITY;
    int bi = 0x7fffffff;
    for (int i = threadIdx.x; i < V; i += blockDim.x) {
        const float v = row[i];
        if (v > best || (v == best && i < bi)) { best = v; bi = i; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
    }
    __shared__ float sv[kWarps];
    __shared__ int si[kWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) { sv[warp] = best; si[warp] = bi; }
    __syncthreads();
    if (warp == 0) {
        best = lane < (blockDim.x >> 5) ? sv[lane] : -INFINITY;
        bi = lane < (blockDim.x >> 5) ? si[lane] : 0x7fffffff;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, best, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
        }
        if (lane == 0) {
            if (bi == 0x7fffffff) bi = 0;   // all NaN: token 0
            out[b] = bi;
            if (tokens_adv) tokens_adv[b] = bi;
            if (pos_adv) pos_adv[b] += 1;
            tl_stamp(tl);
        }
    }
}

// ---------------------------------------------------------------- top-p
// Candidates of the radix select kept in shared memory once the chosen digit
// prefix holds few enough keys: later passes read them instead of the row.
constexpr int kListCap = 4096;

struct TopPShared {
    unsigned long long hist_mass[kWarps][256];
    unsigned int hist_cnt[kWarps][256];
    unsigned long long tot_mass[256];
    unsigned int tot_cnt[256];
    unsigned long long p1_mass[256];     // first-digit histogram of the whole row (both selects start from it)
    unsigned int p1_cnt[256];
    unsigned long long list_key[kListCap];
    unsigned long long list_mass[kListCap];
    unsigned long long red_u64[kWarps];
    float red_f[kWarps];
    unsigned long long sel_prefix, sel_before;
    unsigned int sel_cnt;
    int list_n;
    float lmax;
};

__device__ __forceinline__ unsigned long long fixed_mass(float l, double lmax, double inv_t) {
    const double e = exp((static_cast<double>(l) - lmax) * inv_t);
    return static_cast<unsigned long long>(e * kFixScale + 0.5);
}

// Per-warp histograms of digit (key >> shift) & 255 over the keys that match
// `prefix` under `mask`, from the row (masses computed here) or from the
// candidate list; then the per-digit totals in sh.tot_*.  A thread's
// consecutive keys mostly share a digit: they are summed in registers, one
// pair of shared-memory atomics per change of digit.
__device__ void digit_histogram(TopPShared& sh, const float* row, int V, bool from_list, double lmax, double inv_t,
                                uint64_t prefix, uint64_t mask, int shift) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = lane; i < 256; i += 32) {
        sh.hist_mass[warp][i] = 0ull;
        sh.hist_cnt[warp][i] = 0u;
    }
    __syncthreads();
    int cur = -1;
    unsigned long long cur_mass = 0;
    unsigned int cur_cnt = 0;
    auto add = [&](uint64_t key, unsigned long long m) {
        const int bin = static_cast<int>((key >> shift) & 255u);
        if (bin != cur) {
            if (cur >= 0) {
                atomicAdd(&sh.hist_mass[warp][cur], cur_mass);
                atomicAdd(&sh.hist_cnt[warp][cur], cur_cnt);
            }
            cur = bin;
            cur_mass = 0;
            cur_cnt = 0;
        }
        cur_mass += m;
        ++cur_cnt;
    };
    if (from_list) {
        for (int j = threadIdx.x; j < sh.list_n; j += blockDim.x) {
            const uint64_t key = sh.list_key[j];
            if ((key & mask) == prefix) add(key, sh.list_mass[j]);
        }
    } else {
        for (int i = threadIdx.x; i < V; i += blockDim.x) {
            const float l = row[i];
            const uint64_t key = sort_key(l, i);
            if ((key & mask) == prefix) add(key, fixed_mass(l, lmax, inv_t));
        }
    }
    if (cur >= 0) {
        atomicAdd(&sh.hist_mass[warp][cur], cur_mass);
        atomicAdd(&sh.hist_cnt[warp][cur], cur_cnt);
    }
    __syncthreads();
    if (threadIdx.x < 256) {
        unsigned long long m = 0;
        unsigned int c = 0;
        for (int w = 0; w < kWarps; ++w) {
            m += sh.hist_mass[w][threadIdx.x];
            c += sh.hist_cnt[w][threadIdx.x];
        }
        sh.tot_mass[threadIdx.x] = m;
        sh.tot_cnt[threadIdx.x] = c;
    }
    __syncthreads();
}

// Warp 0: in descending digit order over the totals `tm` / `tc` (256 bins),
// the first digit whose inclusive prefix mass, after `before`, exceeds
// `target` (or the last non-empty digit if none does).  Writes the extended
// prefix, the mass before the chosen digit and its key count to sh.sel_*.
template <typename SH>
__device__ void choose_digit(SH& sh, const unsigned long long* tm, const unsigned int* tc, uint64_t prefix,
                             int shift, unsigned long long before, unsigned long long target) {
    const int lane = threadIdx.x & 31;
    unsigned long long part = 0;
    for (int k = 0; k < 8; ++k) part += tm[255 - 8 * lane - k];   // lane L: digits 255-8L .. 248-8L
    unsigned long long incl = part;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    const unsigned long long excl = incl - part;
    const bool cross = before + incl > target;
    const unsigned int ballot = __ballot_sync(0xffffffffu, cross);
    int chosen = -1;
    unsigned long long chosen_before = 0;
    if (ballot) {
        const int L = __ffs(ballot) - 1;
        if (lane == L) {
            unsigned long long cum = before + excl;
            for (int k = 0; k < 8; ++k) {
                const int bin = 255 - 8 * lane - k;
                if (tc[bin] == 0) continue;
                if (cum + tm[bin] > target) { chosen = bin; chosen_before = cum; break; }
                cum += tm[bin];
            }
        }
        chosen = __shfl_sync(0xffffffffu, chosen, L);
        chosen_before = __shfl_sync(0xffffffffu, chosen_before, L);
    }
    if (chosen < 0) {
        // no digit crosses: the lowest non-empty digit (the last key in order)
        if (lane == 0) {
            unsigned long long cum = before;
            for (int bin = 255; bin >= 0; --bin) {
                if (tc[bin] == 0) continue;
                chosen = bin;
                chosen_before = cum;
                cum += tm[bin];
            }
        }
        chosen = __shfl_sync(0xffffffffu, chosen, 0);
        chosen_before = __shfl_sync(0xffffffffu, chosen_before, 0);
    }
    if (lane == 0) {
        sh.sel_prefix = prefix | (static_cast<uint64_t>(chosen) << shift);
        sh.sel_before = chosen_before;
        sh.sel_cnt = tc[chosen];
    }
}

// The candidates matching `prefix` under `mask` copied from the row into the
// shared list (the caller knows there are at most kListCap of them).
__device__ void compact(TopPShared& sh, const float* row, int V, double lmax, double inv_t, uint64_t prefix,
                        uint64_t mask) {
    if (threadIdx.x == 0) sh.list_n = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < V; i += blockDim.x) {
        const float l = row[i];
        const uint64_t key = sort_key(l, i);
        if ((key & mask) == prefix) {
            const int j = atomicAdd(&sh.list_n, 1);
            sh.list_key[j] = key;
            sh.list_mass[j] = fixed_mass(l, lmax, inv_t);
        }
    }
    __syncthreads();
}

// First key in descending order whose inclusive prefix mass exceeds `target`
// (or the smallest key if none does), starting from the first-digit histogram
// of the whole row (sh.p1_*).  `*list_prefix` names the first-digit prefix
// the shared list holds (or ~0 for none); the list is rebuilt when this select
// chooses another first digit with at most kListCap keys.  Returns the key;
// *before_out = the mass of all keys strictly before it.
__device__ uint64_t radix_select(TopPShared& sh, const float* row, int V, double lmax, double inv_t,
                                 unsigned long long target, uint64_t* list_prefix, unsigned long long* before_out) {
    const int warp = threadIdx.x >> 5;
    if (warp == 0) choose_digit(sh, sh.p1_mass, sh.p1_cnt, 0, 56, 0, target);
    __syncthreads();
    uint64_t prefix = sh.sel_prefix, mask = static_cast<uint64_t>(255) << 56;
    unsigned long long before = sh.sel_before;
    bool use_list = false;
    if (prefix == *list_prefix) {
        use_list = true;
    } else if (sh.sel_cnt <= static_cast<unsigned int>(kListCap)) {
        compact(sh, row, V, lmax, inv_t, prefix, mask);
        *list_prefix = prefix;
        use_list = true;
    }
    __syncthreads();
    for (int pass = 1; pass < 8; ++pass) {
        const int shift = 56 - 8 * pass;
        digit_histogram(sh, row, V, use_list, lmax, inv_t, prefix, mask, shift);
        if (warp == 0) choose_digit(sh, sh.tot_mass, sh.tot_cnt, prefix, shift, before, target);
        __syncthreads();
        prefix = sh.sel_prefix;
        before = sh.sel_before;
        mask |= static_cast<uint64_t>(255) << shift;
        const bool fits = sh.sel_cnt <= static_cast<unsigned int>(kListCap);
        __syncthreads();
        if (!use_list && fits && pass < 7) {
            // few enough keys under the longer prefix: the remaining passes
            // read them from the list (which then serves no other prefix)
            compact(sh, row, V, lmax, inv_t, prefix, mask);
            *list_prefix = ~0ull;
            use_list = true;
        }
    }
    *before_out = before;
    return prefix;
}

__global__ void __launch_bounds__(kSampleThreads)
top_p_kernel(const float* __restrict__ logits, int V, float temperature, float top_p,
             const float* __restrict__ uniforms, int32_t* out, int32_t* tokens_adv, int32_t* pos_adv,
             unsigned long long* tl) {
    extern __shared__ uint8_t smem_raw[];
    TopPShared& sh = *reinterpret_cast<TopPShared*>(smem_raw);
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float* row = logits + static_cast<long long>(b) * V;

    // max logit
    float mx = -INFINITY;
    for (int i = threadIdx.x; i < V; i += blockDim.x) mx = fmaxf(mx, row[i]);
    mx = warp_max(mx);
    if (lane == 0) sh.red_f[warp] = mx;
    __syncthreads();
    if (warp == 0) {
        float t = lane < kWarps ? sh.red_f[lane] : -INFINITY;
        t = warp_max(t);
        if (lane == 0) sh.lmax = t;
    }
    __syncthreads();
    const double lmax = static_cast<double>(sh.lmax);
    const double inv_t = 1.0 / static_cast<double>(temperature);

    // first-digit histogram of the whole row; its digits add up to the row's
    // total mass S (exact integers, so in any order)
    digit_histogram(sh, row, V, false, lmax, inv_t, 0, 0, 56);
    unsigned long long S = 0;
    for (int i = 0; i < 256; ++i) S += sh.tot_mass[i];
    if (threadIdx.x < 256) {
        sh.p1_mass[threadIdx.x] = sh.tot_mass[threadIdx.x];
        sh.p1_cnt[threadIdx.x] = sh.tot_cnt[threadIdx.x];
    }
    __syncthreads();

    // nucleus edge: first key whose inclusive mass exceeds top_p * S
    uint64_t list_prefix = ~0ull;
    const double tp = static_cast<double>(top_p) * static_cast<double>(S);
    const unsigned long long t1 = tp >= 18446744073709549568.0 ? ~0ull : static_cast<unsigned long long>(tp);
    unsigned long long before_edge;
    const uint64_t edge = radix_select(sh, row, V, lmax, inv_t, t1, &list_prefix, &before_edge);
    const int edge_id = static_cast<int>(~static_cast<uint32_t>(edge & 0xffffffffu));
    const unsigned long long Z = before_edge + fixed_mass(row[edge_id], lmax, inv_t);

    // draw: first kept key whose inclusive mass exceeds u * Z
    double u = static_cast<double>(uniforms[b]);
    u = fmin(fmax(u, 0.0), 1.0);
    const unsigned long long t2 = static_cast<unsigned long long>(u * static_cast<double>(Z));
    unsigned long long before_draw;
    const uint64_t drawn = radix_select(sh, row, V, lmax, inv_t, t2, &list_prefix, &before_draw);
    const uint64_t pick = drawn < edge ? edge : drawn;   // never past the nucleus edge
    if (threadIdx.x == 0) {
        const int id = static_cast<int>(~static_cast<uint32_t>(pick & 0xffffffffu));
        out[b] = id;
        if (tokens_adv) tokens_adv[b] = id;
        if (pos_adv) pos_adv[b] += 1;
        tl_stamp(tl);
    }
}

// ---------------------------------------------------------------- top-p on a cluster per row
// The selection of top_p_kernel (same keys, masses, targets and digit rule,
// so the same picks) with each row spread over a cluster of kTpRanks CTAs.
// CTA r owns the contiguous slice [r*S, min(V, (r+1)*S)), S = ceil(V /
// kTpRanks), and keeps its slice's ordered logit bits and fixed-point masses
// in shared memory, so each fp64 exponential is taken once.  Every digit
// histogram is built per CTA and summed over the cluster through distributed
// shared memory; the CTAs then take identical decisions from identical
// integer totals.  Once a digit prefix holds a single key, the CTA that owns
// it publishes the key and the select ends.  Exchanges alternate between two
// buffers, so one cluster barrier per exchange orders every write before the
// reads of the same round and after the reads of two rounds before.
constexpr int kTpRanks = 8;
constexpr int kTpThreads = 512;
constexpr int kTpWarps = kTpThreads / 32;
constexpr int kTpSub = 4;   // shared-memory sub-histograms (warp w adds into sub[w % kTpSub])

struct TpHist {
    unsigned long long mass[256];
    unsigned int cnt[256];
};
struct TpClShared {
    TpHist xh[2];                   // this CTA's digit histogram, read by the cluster
    TpHist sub[kTpSub];
    TpHist tot;                     // cluster totals of the current digit
    TpHist p1;                      // cluster totals of the first digit (both selects start from it)
    unsigned long long xkey[2];     // a key this CTA publishes (0: none; no key is 0)
    unsigned long long sel_prefix, sel_before;
    unsigned int sel_cnt;
    float xmax;                     // this CTA's slice maximum, read by the cluster
    float red_f[kTpWarps];
};
// Behind the struct: uint32_t ob[S] (ordered logit bits), then, 8-byte
// aligned, unsigned long long mass[S].
constexpr size_t kTpFixedBytes = (sizeof(TpClShared) + 15) & ~size_t(15);

__device__ __forceinline__ unsigned long long ld_cluster_u64(uint32_t a) {
    unsigned long long v;
    asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ unsigned int ld_cluster_u32(uint32_t a) {
    unsigned int v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t a) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
    return v;
}

// This CTA's histogram of digit (key >> shift) & 255 over its slice's keys
// that match `prefix` under `mask`, into sh.xh[k].
__device__ void tp_local_hist(TpClShared& sh, const uint32_t* ob, const unsigned long long* mass, int n, int lo,
                              uint64_t prefix, uint64_t mask, int shift, int k) {
    for (int i = threadIdx.x; i < kTpSub * 256; i += blockDim.x) {
        sh.sub[i >> 8].mass[i & 255] = 0ull;
        sh.sub[i >> 8].cnt[i & 255] = 0u;
    }
    __syncthreads();
    TpHist& h = sh.sub[(threadIdx.x >> 5) % kTpSub];
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
        const uint64_t key = (static_cast<uint64_t>(ob[j]) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(lo + j));
        if ((key & mask) == prefix) {
            const int bin = static_cast<int>((key >> shift) & 255u);
            atomicAdd(&h.mass[bin], mass[j]);
            atomicAdd(&h.cnt[bin], 1u);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 256; i += blockDim.x) {
        unsigned long long m = 0;
        unsigned int c = 0;
#pragma unroll
        for (int q = 0; q < kTpSub; ++q) {
            m += sh.sub[q].mass[i];
            c += sh.sub[q].cnt[i];
        }
        sh.xh[k].mass[i] = m;
        sh.xh[k].cnt[i] = c;
    }
}

// sh.tot = the sum over the cluster's CTAs of their sh.xh[k].
__device__ void tp_reduce(TpClShared& sh, int k) {
    cluster_sync();
    for (int i = threadIdx.x; i < 256; i += blockDim.x) {
        unsigned long long m = 0;
        unsigned int c = 0;
#pragma unroll
        for (uint32_t r = 0; r < kTpRanks; ++r) {
            m += ld_cluster_u64(cluster_addr(&sh.xh[k].mass[i], r));
            c += ld_cluster_u32(cluster_addr(&sh.xh[k].cnt[i], r));
        }
        sh.tot.mass[i] = m;
        sh.tot.cnt[i] = c;
    }
    __syncthreads();
}

// First key in descending order whose inclusive prefix mass exceeds
// `target` (or the smallest key if none does), from the first-digit totals
// sh.p1; *before_out = the mass of the keys strictly before it.  `k` is the
// exchange buffer of the next round (advanced here).
__device__ uint64_t tp_select(TpClShared& sh, const uint32_t* ob, const unsigned long long* mass, int n, int lo,
                              unsigned long long target, int& k, unsigned long long* before_out) {
    const int warp = threadIdx.x >> 5;
    if (warp == 0) choose_digit(sh, sh.p1.mass, sh.p1.cnt, 0, 56, 0, target);
    __syncthreads();
    uint64_t prefix = sh.sel_prefix, mask = static_cast<uint64_t>(255) << 56;
    unsigned long long before = sh.sel_before;
    unsigned int cnt = sh.sel_cnt;
    __syncthreads();
    for (int pass = 1; pass < 8 && cnt > 1; ++pass) {
        const int shift = 56 - 8 * pass;
        tp_local_hist(sh, ob, mass, n, lo, prefix, mask, shift, k);
        tp_reduce(sh, k);
        k ^= 1;
        if (warp == 0) choose_digit(sh, sh.tot.mass, sh.tot.cnt, prefix, shift, before, target);
        __syncthreads();
        prefix = sh.sel_prefix;
        before = sh.sel_before;
        cnt = sh.sel_cnt;
        mask |= static_cast<uint64_t>(255) << shift;
        __syncthreads();
    }
    if (mask != ~0ull) {
        // one key under `prefix`: the CTA that owns it publishes it
        if (threadIdx.x == 0) sh.xkey[k] = 0ull;
        __syncthreads();
        for (int j = threadIdx.x; j < n; j += blockDim.x) {
            const uint64_t key =
                (static_cast<uint64_t>(ob[j]) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(lo + j));
            if ((key & mask) == prefix) sh.xkey[k] = key;
        }
        cluster_sync();
        uint64_t key = 0;
#pragma unroll
        for (uint32_t r = 0; r < kTpRanks; ++r) key |= ld_cluster_u64(cluster_addr(&sh.xkey[k], r));
        k ^= 1;
        prefix = key;
    }
    *before_out = before;
    return prefix;
}

__global__ void __cluster_dims__(kTpRanks, 1, 1) __launch_bounds__(kTpThreads, 1)
top_p_cluster_kernel(const float* __restrict__ logits, int V, float temperature, float top_p,
                     const float* __restrict__ uniforms, int32_t* out, int32_t* tokens_adv, int32_t* pos_adv,
                     unsigned long long* tl) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TpClShared& sh = *reinterpret_cast<TpClShared*>(smem_raw);
    pdl_trigger();
    pdl_wait();
    const int rank = static_cast<int>(cluster_rank());
    const int b = blockIdx.x / kTpRanks;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float* row = logits + static_cast<long long>(b) * V;
    const int S = (V + kTpRanks - 1) / kTpRanks;
    const int lo = rank * S;
    const int n = V - lo < S ? (V - lo > 0 ? V - lo : 0) : S;
    uint32_t* ob = reinterpret_cast<uint32_t*>(smem_raw + kTpFixedBytes);
    unsigned long long* mass =
        reinterpret_cast<unsigned long long*>(smem_raw + kTpFixedBytes + ((static_cast<size_t>(S) * 4 + 7) & ~size_t(7)));

    // row maximum: slice maxima, then the cluster's
    float mx = -INFINITY;
    for (int j = threadIdx.x; j < n; j += blockDim.x) mx = fmaxf(mx, row[lo + j]);
    mx = warp_max(mx);
    if (lane == 0) sh.red_f[warp] = mx;
    __syncthreads();
    if (warp == 0) {
        float t = lane < kTpWarps ? sh.red_f[lane] : -INFINITY;
        t = warp_max(t);
        if (lane == 0) sh.xmax = t;
    }
    cluster_sync();
    float lm = -INFINITY;
#pragma unroll
    for (uint32_t r = 0; r < kTpRanks; ++r) lm = fmaxf(lm, ld_cluster_f32(cluster_addr(&sh.xmax, r)));
    const double lmax = static_cast<double>(lm);
    const double inv_t = 1.0 / static_cast<double>(temperature);

    // the slice's keys and masses, once; the first-digit histogram over the cluster
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
        const float l = row[lo + j];
        ob[j] = ordered_bits(l);
        mass[j] = fixed_mass(l, lmax, inv_t);
    }
    __syncthreads();
    int k = 0;
    tp_local_hist(sh, ob, mass, n, lo, 0, 0, 56, k);
    tp_reduce(sh, k);
    k ^= 1;
    unsigned long long S_mass = 0;
    for (int i = 0; i < 256; ++i) S_mass += sh.tot.mass[i];
    for (int i = threadIdx.x; i < 256; i += blockDim.x) {
        sh.p1.mass[i] = sh.tot.mass[i];
        sh.p1.cnt[i] = sh.tot.cnt[i];
    }
    __syncthreads();

    // nucleus edge: first key whose inclusive mass exceeds top_p * S
    const double tp = static_cast<double>(top_p) * static_cast<double>(S_mass);
    const unsigned long long t1 = tp >= 18446744073709549568.0 ? ~0ull : static_cast<unsigned long long>(tp);
    unsigned long long before_edge;
    const uint64_t edge = tp_select(sh, ob, mass, n, lo, t1, k, &before_edge);
    const int edge_id = static_cast<int>(~static_cast<uint32_t>(edge & 0xffffffffu));
    const unsigned long long Z = before_edge + fixed_mass(row[edge_id], lmax, inv_t);

    // draw: first kept key whose inclusive mass exceeds u * Z
    double u = static_cast<double>(uniforms[b]);
    u = fmin(fmax(u, 0.0), 1.0);
    const unsigned long long t2 = static_cast<unsigned long long>(u * static_cast<double>(Z));
    unsigned long long before_draw;
    const uint64_t drawn = tp_select(sh, ob, mass, n, lo, t2, k, &before_draw);
    const uint64_t pick = drawn < edge ? edge : drawn;   // never past the nucleus edge
    if (rank == 0 && threadIdx.x == 0) {
        const int id = static_cast<int>(~static_cast<uint32_t>(pick & 0xffffffffu));
        out[b] = id;
        if (tokens_adv) tokens_adv[b] = id;
        if (pos_adv) pos_adv[b] += 1;
        tl_stamp(tl);
    }
    cluster_sync();   // no CTA leaves while the cluster may still read its shared memory
}

// Vocabularies whose slices fit (V up to about 137k) take the cluster kernel.
constexpr size_t kTpClusterMaxSmem = 227 * 1024;
// Bytes of dynamic shared memory the cluster kernel needs for a vocabulary of V.
static size_t top_p_cluster_smem(int V) {
    const size_t S = static_cast<size_t>((V + kTpRanks - 1) / kTpRanks);
    return kTpFixedBytes + ((S * 4 + 7) & ~size_t(7)) + S * 8;
}

// ---------------------------------------------------------------- token log-probabilities
// out[i] = log softmax(logits[i, :])[tok[i]] = l[tok] - (m + log sum_j exp(l_j - m)),
// m = max_j l_j, the sum in fp64 (the log-probabilities that generate returns,
// Admin Guide §8.5).  An id outside [0, V) gives NaN.
__global__ void __launch_bounds__(kSampleThreads)
logprob_kernel(const float* __restrict__ logits, const int32_t* __restrict__ tok, int V, float* __restrict__ out) {
    __shared__ float s_max[kWarps];
    __shared__ double s_sum[kWarps];
    const int i = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float* row = logits + static_cast<long long>(i) * V;
    float mx = -INFINITY;
    for (int j = threadIdx.x; j < V; j += blockDim.x) mx = fmaxf(mx, row[j]);
    mx = warp_max(mx);
    if (lane == 0) s_max[warp] = mx;
    __syncthreads();
    mx = s_max[0];
    for (int w = 1; w < kWarps; ++w) mx = fmaxf(mx, s_max[w]);
    const double m = static_cast<double>(mx);
    double sum = 0.0;
    for (int j = threadIdx.x; j < V; j += blockDim.x) sum += exp(static_cast<double>(row[j]) - m);
    sum = warp_sum_d(sum);
    if (lane == 0) s_sum[warp] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
        double total = 0.0;
        for (int w = 0; w < kWarps; ++w) total += s_sum[w];
        const int t = tok[i];
        out[i] = (t >= 0 && t < V) ? static_cast<float>(static_cast<double>(row[t]) - m - log(total)) : NAN;
    }
}

int launch_logprobs(const float* logits, const int32_t* tokens, int N, int V, float* out, cudaStream_t st) {
    logprob_kernel<<<N, kSampleThreads, 0, st>>>(logits, tokens, V, out);
    LLB_CHECK_LAUNCH("logprob_kernel");
    return LLAMA_OK;
}

int launch_argmax(const float* logits, int B, int V, int32_t* out, int32_t* tokens_adv, int32_t* pos_adv,
                  cudaStream_t st, bool pdl, unsigned long long* tl) {
    static bool attr = false;
    if (!attr) {
        cudaError_t ce = carveout_max(argmax_kernel);
        if (ce != cudaSuccess) return cuda_fail(ce, "cudaFuncSetAttribute(argmax_kernel)");
        attr = true;
    }
    cudaError_t e = launch_k(argmax_kernel, dim3(B), dim3(kSampleThreads), 0, st, pdl, logits, V, out, tokens_adv,
                             pos_adv, tl);
    count_launch();
    if (e != cudaSuccess) return cuda_fail(e, "argmax_kernel");
    return LLAMA_OK;
}

int launch_top_p(const float* logits, int B, int V, float temperature, float top_p, const float* uniforms,
                 int32_t* out, int32_t* tokens_adv, int32_t* pos_adv, cudaStream_t st, bool pdl,
                 unsigned long long* tl) {
    const size_t csmem = top_p_cluster_smem(V);
    if (csmem <= kTpClusterMaxSmem) {
        static bool cattr = false;
        if (!cattr) {
            cudaError_t e = cudaFuncSetAttribute(top_p_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(kTpClusterMaxSmem));
            if (e == cudaSuccess) e = carveout_max(top_p_cluster_kernel);
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(top_p_cluster_kernel)");
            cattr = true;
        }
        cudaError_t e = launch_k(top_p_cluster_kernel, dim3(B * kTpRanks), dim3(kTpThreads), csmem, st, pdl, logits, V,
                                 temperature, top_p, uniforms, out, tokens_adv, pos_adv, tl);
        count_launch();
        if (e != cudaSuccess) return cuda_fail(e, "top_p_cluster_kernel");
        return LLAMA_OK;
    }
    const int smem = static_cast<int>(sizeof(TopPShared));
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(top_p_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess) e = carveout_max(top_p_kernel);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(top_p_kernel)");
        attr = true;
    }
    cudaError_t e = launch_k(top_p_kernel, dim3(B), dim3(kSampleThreads), smem, st, pdl, logits, V, temperature,
                             top_p, uniforms, out, tokens_adv, pos_adv, tl);
    count_launch();
    if (e != cudaSuccess) return cuda_fail(e, "top_p_kernel");
    return LLAMA_OK;
}

}  // namespace llb
