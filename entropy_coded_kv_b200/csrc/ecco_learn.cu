// Table learner: one tensor's patterns and codebooks from a bf16 sample in
// device memory.
//
// The review page ("Ecco: Improving Memory Bandwidth and Capacity for LLMs via
// Entropy-aware Cache Compression", "What carries the argument" and the free
// parameters) fixes what is learned -- 64 shared patterns of 15 sorted
// centroids per tensor, 4 Huffman codebooks per pattern with lengths of at
// most 8 bits (referee comment 1) -- but not how.  The construction is the
// library's own (the same steps as the host learner entropy_coded_kv_b200/calib.py):
//   1. S_t = absmax(sample) / 448 (the per-tensor FP8 factor, Fig. 4 caption).
//   2. Each sampled group is scaled by its FP8 group scale; the element of
//      largest magnitude is set aside; the remaining values, sorted, are
//      summarised by 15 equal-count bin means.
//   3. k-means (k-means++ seeding, 20 Lloyd iterations) over those 15-vectors
//      gives the initial patterns.
//   4. 4 refinement rounds in the encoder's own terms: groups go to patterns by
//      the min/max rule, values to centroids by the thresholds, and every
//      centroid moves to the mean of its values.
//   5. Per pattern, the groups' symbol histograms are split into 4 clusters; each
//      cluster gets an optimal length-limited prefix code (package-merge,
//      Larmore & Hirschberg 1990, lengths <= 8, every symbol codable), and groups
//      move to the codebook that codes them shortest (6 rounds).
// The data-parallel parts (absmax, per-group scaling and sorting, k-means
// assignment, refinement sums, histograms) are CUDA kernels; the small serial
// parts (seeding, centroid means, package-merge, codebook clustering) run on
// the host.  Sums over groups are formed in a fixed order, so a given sample
// and seed always give the same blob.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <unordered_set>
#include <vector>

#include "ecco_internal.cuh"

namespace ecco {
namespace {

constexpr int kMaxSample = 16384;  // sampled groups
constexpr int kLloydIters = 20;
constexpr int kRefineRounds = 4;
constexpr int kBookRounds = 6;
constexpr int kBookLloyd = 10;
constexpr int kLearnWarps = 8;  // warps per CTA of the per-group kernels

// splitmix64 (Steele, Lea, Flood 2014): the learner's seeded random stream.
struct Rng {
    uint64_t s;
    uint64_t next()
    {
        uint64_t z = (s += 0x9E3779B97F4A7C15ull);
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        return z ^ (z >> 31);
    }
    double uniform() { return (double)(next() >> 11) * (1.0 / 9007199254740992.0); }
    int64_t below(int64_t n) { return (int64_t)(next() % (uint64_t)n); }
};

struct Edges {
    int e[16];  // bin b of the sorted remaining values: [e[b], e[b+1])
};

// ------------------------------------------------------------------ kernels
__global__ void absmax_kernel(const uint16_t* __restrict__ x, int64_t n, unsigned int* out)
{
    unsigned int best = 0;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const unsigned int v = x[i] & 0x7fffu;
        if (v < 0x7f80u) best = max(best, v);  // finite values only
    }
    best = __reduce_max_sync(0xffffffffu, best);
    if ((threadIdx.x & 31) == 0) atomicMax(out, best);
}

// One warp per sampled group: scale, normalise, sort the remaining values,
// 15 bin means, min / max.  Lane l holds elements l*V .. l*V+V-1.
template <int G>
__global__ void __launch_bounds__(kLearnWarps * 32) features_kernel(
    const uint16_t* __restrict__ x, const int64_t* __restrict__ idx, int n, float S_t, Edges E,
    float* __restrict__ u_out, float* __restrict__ F, float* __restrict__ umin_out, float* __restrict__ umax_out,
    int* __restrict__ m_out, int* __restrict__ keep_out)
{
    constexpr int V = G / 32;
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kLearnWarps + (threadIdx.x >> 5);
    if (gw >= n) return;
    const uint16_t* src = x + idx[gw] * G + lane * V;
    uint32_t b[V];
#pragma unroll
    for (int r = 0; r < V; ++r) {
        b[r] = src[r];
        if ((b[r] & 0x7f80u) == 0x7f80u) b[r] = 0;  // non-finite -> +0
    }
    // first index of the largest magnitude, with its sign
    uint32_t key = 0;
#pragma unroll
    for (int r = 0; r < V; ++r)
        key = max(key, ((b[r] & 0x7fffu) << 8) | ((uint32_t)(127 - (lane * V + r)) << 1) | (b[r] >> 15));
    key = __reduce_max_sync(0xffffffffu, key);
    const int m = 127 - (int)((key >> 1) & 127u);
    const float xm_abs = __uint_as_float((key >> 8) << 16);
    const uint32_t code = (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(xm_abs, S_t), __NV_SATFINITE, __NV_E4M3);
    const float s_abs = __fmul_rn(S_t, e4m3_to_f32(code & 0x7fu));
    const int keep = s_abs != 0.0f;
    const float s = (key & 1u) ? -s_abs : s_abs;
    const float inv = keep ? __frcp_rn(s) : 0.0f;
    float v[V];
    float lmin = INFINITY, lmax = -INFINITY;
#pragma unroll
    for (int r = 0; r < V; ++r) {
        const int k = lane * V + r;
        const float uk = (k == m) ? 0.0f : __fmul_rn(bf16_bits_to_f32(b[r]), inv);
        u_out[(int64_t)gw * G + k] = uk;
        if (k != m) {
            lmin = fminf(lmin, uk);
            lmax = fmaxf(lmax, uk);
        }
        v[r] = (k == m) ? INFINITY : uk;  // the scale element sorts last
    }
    // bitonic sort, ascending, element k = lane * V + r
#pragma unroll
    for (int size = 2; size <= G; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            if (stride < V) {
#pragma unroll
                for (int r = 0; r < V; ++r) {
                    const int rp = r ^ stride;
                    if (rp > r) {
                        const bool asc = ((lane * V + r) & size) == 0;
                        const float lo = fminf(v[r], v[rp]), hi = fmaxf(v[r], v[rp]);
                        v[r] = asc ? lo : hi;
                        v[rp] = asc ? hi : lo;
                    }
                }
            } else {
#pragma unroll
                for (int r = 0; r < V; ++r) {
                    const int k = lane * V + r;
                    const float vp = __shfl_xor_sync(0xffffffffu, v[r], stride / V);
                    const bool asc = (k & size) == 0;
                    const bool keep_min = ((k & stride) == 0) == asc;
                    v[r] = keep_min ? fminf(v[r], vp) : fmaxf(v[r], vp);
                }
            }
        }
    }
    // bin means
#pragma unroll 1
    for (int j = 0; j < kNCent; ++j) {
        float part = 0.0f;
#pragma unroll
        for (int r = 0; r < V; ++r) {
            const int k = lane * V + r;
            if (k >= E.e[j] && k < E.e[j + 1]) part += v[r];
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == 0) F[(int64_t)gw * kNCent + j] = part / (float)(E.e[j + 1] - E.e[j]);
    }
    lmin = warp_min_f32(lmin);
    lmax = warp_max_f32(lmax);
    if (lane == 0) {
        umin_out[gw] = lmin;
        umax_out[gw] = lmax;
        m_out[gw] = m;
        keep_out[gw] = keep;
    }
}

// Thread per point: nearest of k centres (squared distance, first of ties).
__global__ void assign_kernel(const float* __restrict__ F, int n, const float* __restrict__ Cin, int k,
                              int* __restrict__ a)
{
    __shared__ float C[kNPat * kNCent];
    for (int i = threadIdx.x; i < k * kNCent; i += blockDim.x) C[i] = Cin[i];
    __syncthreads();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float f[kNCent];
#pragma unroll
    for (int j = 0; j < kNCent; ++j) f[j] = F[(int64_t)i * kNCent + j];
    float best = INFINITY;
    int bi = 0;
    for (int c = 0; c < k; ++c) {
        float d = 0.0f;
#pragma unroll
        for (int j = 0; j < kNCent; ++j) {
            const float t = f[j] - C[c * kNCent + j];
            d = fmaf(t, t, d);
        }
        if (d < best) {
            best = d;
            bi = c;
        }
    }
    a[i] = bi;
}

// Warp per group: pattern by the min/max rule (R8), symbols by the thresholds
// (R9), per-(pattern, symbol) sums of the values and counts.  Each warp adds
// its groups in order into its own shared-memory rows; the CTA then writes
// the sum of its warps, in warp order, to part_sum / part_cnt [CTA][64][15].
template <int G>
__global__ void __launch_bounds__(kLearnWarps * 32) refine_kernel(
    const float* __restrict__ u, const int* __restrict__ m_in, const float* __restrict__ umin,
    const float* __restrict__ umax, int n, const float* __restrict__ Cin, int npat, double* __restrict__ part_sum,
    int* __restrict__ part_cnt, int* __restrict__ p_out, int* __restrict__ hist)
{
    constexpr int V = G / 32;
    extern __shared__ __align__(16) uint8_t smem[];
    double* acc = reinterpret_cast<double*>(smem);                         // [warp][64][15]
    int* cnt = reinterpret_cast<int*>(acc + kLearnWarps * kNPat * kNCent);  // [warp][64][15]
    float* C = reinterpret_cast<float*>(cnt + kLearnWarps * kNPat * kNCent);  // [64][15]
    float* T = C + kNPat * kNCent;                                          // [64][14]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < kLearnWarps * kNPat * kNCent; i += blockDim.x) {
        acc[i] = 0.0;
        cnt[i] = 0;
    }
    for (int i = tid; i < kNPat * kNCent; i += blockDim.x) C[i] = Cin[i];
    __syncthreads();
    for (int i = tid; i < kNPat * (kNCent - 1); i += blockDim.x) {
        const int q = i / (kNCent - 1), j = i - q * (kNCent - 1);
        T[i] = __fmul_rn(__fadd_rn(C[q * kNCent + j], C[q * kNCent + j + 1]), 0.5f);
    }
    __syncthreads();
    double* wacc = acc + warp * kNPat * kNCent;
    int* wcnt = cnt + warp * kNPat * kNCent;
    const int nwarps = gridDim.x * kLearnWarps;
    for (int g = blockIdx.x * kLearnWarps + warp; g < n; g += nwarps) {
        const float lo = umin[g], hi = umax[g];
        // min/max pattern: lane evaluates q = lane, lane + 32
        uint32_t eb = 0xffffffffu, bq = 64u;
        for (int q = lane; q < npat; q += 32) {
            const float d0 = __fsub_rn(lo, C[q * kNCent]), d1 = __fsub_rn(hi, C[q * kNCent + kNCent - 1]);
            const uint32_t e = __float_as_uint(__fadd_rn(__fmul_rn(d0, d0), __fmul_rn(d1, d1)));
            if (e < eb) {
                eb = e;
                bq = (uint32_t)q;
            }
        }
        const uint32_t emin = __reduce_min_sync(0xffffffffu, eb);
        const int p = (int)__reduce_min_sync(0xffffffffu, eb == emin ? bq : 64u);
        const int m = m_in[g];
        int sym[V];
        float val[V];
#pragma unroll
        for (int r = 0; r < V; ++r) {
            const int k = lane * V + r;
            val[r] = u[(int64_t)g * G + k];
            int sy = 0;
#pragma unroll
            for (int j = 0; j < kNCent - 1; ++j) sy += (val[r] > T[p * (kNCent - 1) + j]) ? 1 : 0;
            sym[r] = (k == m) ? 15 : sy;
        }
#pragma unroll 1
        for (int j = 0; j < kNCent; ++j) {
            double sj = 0.0;
            int cj = 0;
#pragma unroll
            for (int r = 0; r < V; ++r)
                if (sym[r] == j) {
                    sj += (double)val[r];
                    ++cj;
                }
#pragma unroll
            for (int o = 16; o; o >>= 1) sj += __shfl_xor_sync(0xffffffffu, sj, o);
            cj = __reduce_add_sync(0xffffffffu, cj);
            if (lane == 0) {
                wacc[p * kNCent + j] += sj;
                wcnt[p * kNCent + j] += cj;
                if (hist) hist[(int64_t)g * kNSym + j] = cj;
            }
        }
        if (lane == 0) {
            if (hist) hist[(int64_t)g * kNSym + 15] = 1;
            if (p_out) p_out[g] = p;
        }
    }
    __syncthreads();
    for (int i = tid; i < kNPat * kNCent; i += blockDim.x) {
        double s = 0.0;
        int c = 0;
        for (int w = 0; w < kLearnWarps; ++w) {
            s += acc[w * kNPat * kNCent + i];
            c += cnt[w * kNPat * kNCent + i];
        }
        part_sum[(int64_t)blockIdx.x * kNPat * kNCent + i] = s;
        part_cnt[(int64_t)blockIdx.x * kNPat * kNCent + i] = c;
    }
}

constexpr size_t kRefineSmem = (size_t)kLearnWarps * kNPat * kNCent * (8 + 4) + (size_t)kNPat * kNCent * 4 +
                               (size_t)kNPat * (kNCent - 1) * 4;

// ------------------------------------------------------------------ host helpers
struct DevBuf {
    void* p = nullptr;
    ~DevBuf()
    {
        if (p) cudaFree(p);
    }
    cudaError_t alloc(size_t n) { return cudaMalloc(&p, n > 0 ? n : 1); }
    template <class T>
    T* as() const
    {
        return static_cast<T*>(p);
    }
};

std::vector<float> strictly_increasing(const double* c)
{
    std::vector<float> v(kNCent);
    for (int j = 0; j < kNCent; ++j) v[j] = (float)std::min(4.0, std::max(-4.0, c[j]));
    std::sort(v.begin(), v.end());
    for (int j = 1; j < kNCent; ++j)
        if (!(v[j] > v[j - 1])) v[j] = std::nextafter(v[j - 1], INFINITY);
    return v;
}

void kmeans_pp(const std::vector<double>& P, int n, int d, int k, Rng& rng, std::vector<double>& C)
{
    C.assign((size_t)k * d, 0.0);
    std::vector<double> d2(n);
    int64_t first = rng.below(n);
    std::copy(&P[first * d], &P[first * d] + d, &C[0]);
    for (int i = 0; i < n; ++i) {
        double t = 0;
        for (int j = 0; j < d; ++j) t += (P[(size_t)i * d + j] - C[j]) * (P[(size_t)i * d + j] - C[j]);
        d2[i] = t;
    }
    for (int c = 1; c < k; ++c) {
        double tot = 0;
        for (int i = 0; i < n; ++i) tot += d2[i];
        int64_t pick;
        if (tot <= 0) {
            pick = rng.below(n);
        } else {
            double r = rng.uniform() * tot, run = 0;
            pick = n - 1;
            for (int i = 0; i < n; ++i) {
                run += d2[i];
                if (run > r) {
                    pick = i;
                    break;
                }
            }
        }
        std::copy(&P[pick * d], &P[pick * d] + d, &C[(size_t)c * d]);
        for (int i = 0; i < n; ++i) {
            double t = 0;
            for (int j = 0; j < d; ++j)
                t += (P[(size_t)i * d + j] - C[(size_t)c * d + j]) * (P[(size_t)i * d + j] - C[(size_t)c * d + j]);
            d2[i] = std::min(d2[i], t);
        }
    }
}

int nearest(const double* p, const std::vector<double>& C, int k, int d)
{
    double best = INFINITY;
    int bi = 0;
    for (int c = 0; c < k; ++c) {
        double t = 0;
        for (int j = 0; j < d; ++j) t += (p[j] - C[(size_t)c * d + j]) * (p[j] - C[(size_t)c * d + j]);
        if (t < best) {
            best = t;
            bi = c;
        }
    }
    return bi;
}

}  // namespace

// Optimal prefix-code lengths with every length <= max_len (package-merge:
// coins of every length level are the symbols; pairs of the cheapest items
// are packaged level by level; a symbol's length is the number of the 2n - 2
// cheapest final items that contain it).  Ties keep the sorted order.
int huffman_lengths(const double* w, int n, int max_len, uint8_t* lens)
{
    if (n < 1 || max_len < 1 || max_len > 30 || (n > 1 && n > (1 << std::min(max_len, 30)))) return -1;
    if (n == 1) {
        lens[0] = 1;
        return 0;
    }
    struct Item {
        double w;
        std::vector<int> syms;
    };
    std::vector<int> order(n);
    for (int i = 0; i < n; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return w[a] < w[b]; });
    std::vector<Item> leaves;
    for (int i : order) leaves.push_back({w[i], {i}});
    std::vector<Item> cur = leaves;
    for (int level = 1; level < max_len; ++level) {
        std::vector<Item> pk;
        for (size_t k = 0; k + 1 < cur.size(); k += 2) {
            Item it{cur[k].w + cur[k + 1].w, cur[k].syms};
            it.syms.insert(it.syms.end(), cur[k + 1].syms.begin(), cur[k + 1].syms.end());
            pk.push_back(std::move(it));
        }
        std::vector<Item> merged;
        size_t a = 0, b = 0;
        while (a < leaves.size() || b < pk.size()) {
            if (b >= pk.size() || (a < leaves.size() && leaves[a].w <= pk[b].w))
                merged.push_back(leaves[a++]);
            else
                merged.push_back(pk[b++]);
        }
        cur = std::move(merged);
    }
    std::vector<int> L(n, 0);
    for (size_t k = 0; k < (size_t)(2 * n - 2) && k < cur.size(); ++k)
        for (int s : cur[k].syms) L[s] += 1;
    for (int i = 0; i < n; ++i) lens[i] = (uint8_t)L[i];
    return 0;
}

cudaError_t learn_tables(const uint16_t* x, int64_t n_groups, int G, int npat, uint64_t seed, uint8_t* blob,
                         cudaStream_t s)
{
    Rng rng{seed};
    // 1. S_t from the absmax of every finite value
    DevBuf d_amax;
    cudaError_t e = d_amax.alloc(sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    cudaMemsetAsync(d_amax.p, 0, sizeof(unsigned int), s);
    const int64_t nval = n_groups * G;
    absmax_kernel<<<(int)std::min<int64_t>((nval + 255) / 256, 4096), 256, 0, s>>>(x, nval, d_amax.as<unsigned int>());
    unsigned int amax_bits = 0;
    if ((e = cudaMemcpyAsync(&amax_bits, d_amax.p, 4, cudaMemcpyDeviceToHost, s)) != cudaSuccess) return e;
    if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return e;
    float amax;
    {
        uint32_t f = amax_bits << 16;
        std::memcpy(&amax, &f, 4);
    }
    float S_t = amax > 0.0f ? amax / 448.0f : 1.0f;
    S_t = std::min(std::max(S_t, std::ldexp(1.0f, -60)), std::ldexp(1.0f, 60));

    // 2. sample (sorted, without replacement), features of the kept groups
    std::vector<int64_t> sel;
    if (n_groups > kMaxSample) {  // Floyd's algorithm: kMaxSample distinct indexes, O(kMaxSample) memory
        std::unordered_set<int64_t> taken;
        taken.reserve(2 * kMaxSample);
        for (int64_t j = n_groups - kMaxSample; j < n_groups; ++j) {
            const int64_t t = rng.below(j + 1);
            taken.insert(taken.count(t) ? j : t);
        }
        sel.assign(taken.begin(), taken.end());
        std::sort(sel.begin(), sel.end());
    } else {
        sel.resize(n_groups);
        for (int64_t i = 0; i < n_groups; ++i) sel[i] = i;
    }
    Edges E;
    for (int j = 0; j <= kNCent; ++j) E.e[j] = (int)std::nearbyint((double)(G - 1) * j / kNCent);
    const int ns = (int)sel.size();
    const int cap = std::max(ns, npat + 1);
    DevBuf d_idx, d_u, d_F, d_lo, d_hi, d_m, d_keep, d_a;
    if ((e = d_idx.alloc(sizeof(int64_t) * cap)) || (e = d_u.alloc(sizeof(float) * cap * G)) ||
        (e = d_F.alloc(sizeof(float) * cap * kNCent)) || (e = d_lo.alloc(sizeof(float) * cap)) ||
        (e = d_hi.alloc(sizeof(float) * cap)) || (e = d_m.alloc(sizeof(int) * cap)) ||
        (e = d_keep.alloc(sizeof(int) * cap)) || (e = d_a.alloc(sizeof(int) * cap)))
        return e;
    auto run_features = [&](int count) {
        const int blocks = (count + kLearnWarps - 1) / kLearnWarps;
        if (count == 0) return;
        if (G == kG)
            features_kernel<kG><<<blocks, kLearnWarps * 32, 0, s>>>(x, d_idx.as<int64_t>(), count, S_t, E, d_u.as<float>(),
                                                                     d_F.as<float>(), d_lo.as<float>(), d_hi.as<float>(),
                                                                     d_m.as<int>(), d_keep.as<int>());
        else
            features_kernel<kGAct><<<blocks, kLearnWarps * 32, 0, s>>>(
                x, d_idx.as<int64_t>(), count, S_t, E, d_u.as<float>(), d_F.as<float>(), d_lo.as<float>(),
                d_hi.as<float>(), d_m.as<int>(), d_keep.as<int>());
    };
    if ((e = cudaMemcpyAsync(d_idx.p, sel.data(), sizeof(int64_t) * ns, cudaMemcpyHostToDevice, s))) return e;
    run_features(ns);
    std::vector<int> keep(ns);
    if ((e = cudaMemcpyAsync(keep.data(), d_keep.p, sizeof(int) * ns, cudaMemcpyDeviceToHost, s))) return e;
    if ((e = cudaStreamSynchronize(s))) return e;
    std::vector<int64_t> kept;
    for (int i = 0; i < ns; ++i)
        if (keep[i]) kept.push_back(sel[i]);
    int n = (int)kept.size();
    if (n != ns) {  // features again on the kept groups only
        if ((e = cudaMemcpyAsync(d_idx.p, kept.data(), sizeof(int64_t) * n, cudaMemcpyHostToDevice, s))) return e;
        run_features(n);
    }
    if (n < npat) {  // too few groups: pad with all-zero groups
        const int pad = npat + 1 - n;
        cudaMemsetAsync(d_u.as<float>() + (int64_t)n * G, 0, sizeof(float) * pad * G, s);
        cudaMemsetAsync(d_F.as<float>() + (int64_t)n * kNCent, 0, sizeof(float) * pad * kNCent, s);
        cudaMemsetAsync(d_lo.as<float>() + n, 0, sizeof(float) * pad, s);
        cudaMemsetAsync(d_hi.as<float>() + n, 0, sizeof(float) * pad, s);
        cudaMemsetAsync(d_m.as<int>() + n, 0, sizeof(int) * pad, s);
        n += pad;
    }
    if ((e = cudaGetLastError())) return e;
    std::vector<float> Ff((size_t)n * kNCent);
    if ((e = cudaMemcpyAsync(Ff.data(), d_F.p, sizeof(float) * Ff.size(), cudaMemcpyDeviceToHost, s))) return e;
    if ((e = cudaStreamSynchronize(s))) return e;
    std::vector<double> F(Ff.begin(), Ff.end());

    // 3. k-means over the 15-vectors: seeding on the host, assignment on the GPU
    std::vector<double> Cd;
    kmeans_pp(F, n, kNCent, npat, rng, Cd);
    std::vector<float> Cf((size_t)kNPat * kNCent, 0.0f);
    std::vector<int> a(n);
    DevBuf d_C;
    if ((e = d_C.alloc(sizeof(float) * kNPat * kNCent))) return e;
    for (int it = 0; it < kLloydIters; ++it) {
        for (size_t i = 0; i < (size_t)npat * kNCent; ++i) Cf[i] = (float)Cd[i];
        if ((e = cudaMemcpyAsync(d_C.p, Cf.data(), sizeof(float) * npat * kNCent, cudaMemcpyHostToDevice, s)))
            return e;
        assign_kernel<<<(n + 255) / 256, 256, 0, s>>>(d_F.as<float>(), n, d_C.as<float>(), npat, d_a.as<int>());
        if ((e = cudaMemcpyAsync(a.data(), d_a.p, sizeof(int) * n, cudaMemcpyDeviceToHost, s))) return e;
        if ((e = cudaStreamSynchronize(s))) return e;
        std::vector<double> sum((size_t)npat * kNCent, 0.0);
        std::vector<int> cnt(npat, 0);
        for (int i = 0; i < n; ++i) {
            cnt[a[i]] += 1;
            for (int j = 0; j < kNCent; ++j) sum[(size_t)a[i] * kNCent + j] += F[(size_t)i * kNCent + j];
        }
        for (int c = 0; c < npat; ++c) {
            if (cnt[c]) {
                for (int j = 0; j < kNCent; ++j) Cd[(size_t)c * kNCent + j] = sum[(size_t)c * kNCent + j] / cnt[c];
            } else {
                const int64_t r = rng.below(n);
                for (int j = 0; j < kNCent; ++j) Cd[(size_t)c * kNCent + j] = F[(size_t)r * kNCent + j];
            }
        }
    }
    std::vector<float> C((size_t)kNPat * kNCent, 0.0f);
    for (int c = 0; c < npat; ++c) {
        std::vector<float> v = strictly_increasing(&Cd[(size_t)c * kNCent]);
        std::copy(v.begin(), v.end(), &C[(size_t)c * kNCent]);
    }

    // 4. refinement in the encoder's terms; 5. final assignment and histograms
    const int rblocks = std::min((n + kLearnWarps - 1) / kLearnWarps, 4 * device_sm_count());
    DevBuf d_ps, d_pc, d_p, d_hist;
    if ((e = d_ps.alloc(sizeof(double) * rblocks * kNPat * kNCent)) ||
        (e = d_pc.alloc(sizeof(int) * rblocks * kNPat * kNCent)) || (e = d_p.alloc(sizeof(int) * n)) ||
        (e = d_hist.alloc(sizeof(int) * (size_t)n * kNSym)))
        return e;
    {
        static std::atomic<uint64_t> done_g{0}, done_a{0};
        cudaError_t ea = set_max_smem_once(done_g, (const void*)refine_kernel<kG>, kRefineSmem);
        cudaError_t eb = set_max_smem_once(done_a, (const void*)refine_kernel<kGAct>, kRefineSmem);
        if (ea != cudaSuccess) return ea;
        if (eb != cudaSuccess) return eb;
    }
    std::vector<double> ps((size_t)rblocks * kNPat * kNCent);
    std::vector<int> pc((size_t)rblocks * kNPat * kNCent);
    for (int round = 0; round <= kRefineRounds; ++round) {
        const bool last = round == kRefineRounds;
        if ((e = cudaMemcpyAsync(d_C.p, C.data(), sizeof(float) * kNPat * kNCent, cudaMemcpyHostToDevice, s)))
            return e;
        if (G == kG)
            refine_kernel<kG><<<rblocks, kLearnWarps * 32, kRefineSmem, s>>>(
                d_u.as<float>(), d_m.as<int>(), d_lo.as<float>(), d_hi.as<float>(), n, d_C.as<float>(), npat,
                d_ps.as<double>(), d_pc.as<int>(), last ? d_p.as<int>() : nullptr, last ? d_hist.as<int>() : nullptr);
        else
            refine_kernel<kGAct><<<rblocks, kLearnWarps * 32, kRefineSmem, s>>>(
                d_u.as<float>(), d_m.as<int>(), d_lo.as<float>(), d_hi.as<float>(), n, d_C.as<float>(), npat,
                d_ps.as<double>(), d_pc.as<int>(), last ? d_p.as<int>() : nullptr, last ? d_hist.as<int>() : nullptr);
        if ((e = cudaGetLastError())) return e;
        if (last) break;
        if ((e = cudaMemcpyAsync(ps.data(), d_ps.p, sizeof(double) * ps.size(), cudaMemcpyDeviceToHost, s))) return e;
        if ((e = cudaMemcpyAsync(pc.data(), d_pc.p, sizeof(int) * pc.size(), cudaMemcpyDeviceToHost, s))) return e;
        if ((e = cudaStreamSynchronize(s))) return e;
        for (int q = 0; q < npat; ++q) {
            double newc[kNCent];
            for (int j = 0; j < kNCent; ++j) {
                double sj = 0.0;
                long long cj = 0;
                for (int b = 0; b < rblocks; ++b) {
                    sj += ps[((size_t)b * kNPat + q) * kNCent + j];
                    cj += pc[((size_t)b * kNPat + q) * kNCent + j];
                }
                newc[j] = cj > 0 ? sj / (double)cj : (double)C[(size_t)q * kNCent + j];
            }
            bool any = false;
            for (int b = 0; b < rblocks && !any; ++b)
                for (int j = 0; j < kNCent && !any; ++j) any = pc[((size_t)b * kNPat + q) * kNCent + j] > 0;
            if (!any) continue;  // no group chose this pattern: unchanged
            std::vector<float> v = strictly_increasing(newc);
            std::copy(v.begin(), v.end(), &C[(size_t)q * kNCent]);
        }
    }
    std::vector<int> pg(n), hist((size_t)n * kNSym);
    if ((e = cudaMemcpyAsync(pg.data(), d_p.p, sizeof(int) * n, cudaMemcpyDeviceToHost, s))) return e;
    if ((e = cudaMemcpyAsync(hist.data(), d_hist.p, sizeof(int) * hist.size(), cudaMemcpyDeviceToHost, s))) return e;
    if ((e = cudaStreamSynchronize(s))) return e;

    // codebooks per pattern
    std::vector<uint8_t> lens((size_t)kNPat * kNBook * kNSym);
    uint8_t glob[kNSym];
    {
        double wsum[kNSym] = {0};
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < kNSym; ++j) wsum[j] += hist[(size_t)i * kNSym + j];
        for (int j = 0; j < kNSym; ++j) wsum[j] += 1.0;
        huffman_lengths(wsum, kNSym, kLMax, glob);
    }
    for (int q = 0; q < npat; ++q) {
        std::vector<int> members;
        for (int i = 0; i < n; ++i)
            if (pg[i] == q) members.push_back(i);
        uint8_t* Lq = &lens[(size_t)q * kNBook * kNSym];
        if (members.empty()) {
            for (int h = 0; h < kNBook; ++h) std::copy(glob, glob + kNSym, Lq + h * kNSym);
            continue;
        }
        double base[kNSym] = {0};
        for (int i : members)
            for (int j = 0; j < kNSym; ++j) base[j] += hist[(size_t)i * kNSym + j];
        for (int j = 0; j < kNSym; ++j) base[j] += 1.0;
        if ((int)members.size() < kNBook) {
            uint8_t l[kNSym];
            huffman_lengths(base, kNSym, kLMax, l);
            for (int h = 0; h < kNBook; ++h) std::copy(l, l + kNSym, Lq + h * kNSym);
            continue;
        }
        const int nm = (int)members.size();
        std::vector<double> P((size_t)nm * kNSym);
        for (int t = 0; t < nm; ++t) {
            double tot = 0;
            for (int j = 0; j < kNSym; ++j) tot += hist[(size_t)members[t] * kNSym + j];
            for (int j = 0; j < kNSym; ++j) P[(size_t)t * kNSym + j] = hist[(size_t)members[t] * kNSym + j] / tot;
        }
        std::vector<double> cen;
        kmeans_pp(P, nm, kNSym, kNBook, rng, cen);
        std::vector<int> asg(nm);
        for (int it = 0; it < kBookLloyd; ++it) {
            for (int t = 0; t < nm; ++t) asg[t] = nearest(&P[(size_t)t * kNSym], cen, kNBook, kNSym);
            for (int c = 0; c < kNBook; ++c) {
                int cc = 0;
                std::vector<double> sm(kNSym, 0.0);
                for (int t = 0; t < nm; ++t)
                    if (asg[t] == c) {
                        ++cc;
                        for (int j = 0; j < kNSym; ++j) sm[j] += P[(size_t)t * kNSym + j];
                    }
                if (cc)
                    for (int j = 0; j < kNSym; ++j) cen[(size_t)c * kNSym + j] = sm[j] / cc;
                else {
                    const int64_t r = rng.below(nm);
                    for (int j = 0; j < kNSym; ++j) cen[(size_t)c * kNSym + j] = P[(size_t)r * kNSym + j];
                }
            }
        }
        for (int t = 0; t < nm; ++t) asg[t] = nearest(&P[(size_t)t * kNSym], cen, kNBook, kNSym);
        uint8_t books[kNBook][kNSym];
        for (int round = 0; round < kBookRounds; ++round) {
            for (int h = 0; h < kNBook; ++h) {
                double wsum[kNSym] = {0};
                bool any = false;
                for (int t = 0; t < nm; ++t)
                    if (asg[t] == h) {
                        any = true;
                        for (int j = 0; j < kNSym; ++j) wsum[j] += hist[(size_t)members[t] * kNSym + j];
                    }
                for (int j = 0; j < kNSym; ++j) wsum[j] = any ? wsum[j] + 1.0 : base[j];
                huffman_lengths(wsum, kNSym, kLMax, books[h]);
            }
            for (int t = 0; t < nm; ++t) {
                long long best = -1;
                int bh = 0;
                for (int h = 0; h < kNBook; ++h) {
                    long long bits = 0;
                    for (int j = 0; j < kNSym; ++j) bits += (long long)hist[(size_t)members[t] * kNSym + j] * books[h][j];
                    if (best < 0 || bits < best) {
                        best = bits;
                        bh = h;
                    }
                }
                asg[t] = bh;
            }
        }
        for (int h = 0; h < kNBook; ++h) std::copy(books[h], books[h] + kNSym, Lq + h * kNSym);
    }
    for (int q = npat; q < kNPat; ++q) {  // unused rows repeat row 0
        std::copy(&C[0], &C[kNCent], &C[(size_t)q * kNCent]);
        std::copy(&lens[0], &lens[kNBook * kNSym], &lens[(size_t)q * kNBook * kNSym]);
    }

    // blob: magic, version, S_t, reserved, C[64][15] f32, len[64][4][16] u8
    uint32_t hdr[4] = {ECCO_TABLES_MAGIC, 1u, 0u, 0u};
    std::memcpy(&hdr[2], &S_t, 4);
    std::memcpy(blob, hdr, 16);
    std::memcpy(blob + 16, C.data(), sizeof(float) * kNPat * kNCent);
    std::memcpy(blob + 16 + sizeof(float) * kNPat * kNCent, lens.data(), lens.size());
    return cudaSuccess;
}

}  // namespace ecco
