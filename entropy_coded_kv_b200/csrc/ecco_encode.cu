// Encoder: one warp per 128-value group, lane l owning values 4l..4l+3.
//
// Steps ("Ecco: Improving Memory Bandwidth and Capacity for LLMs via
// Entropy-aware Cache Compression", review page):
//   scale     per-group FP8 scale from the per-tensor factor (Fig. 4 caption),
//   normalise values divided by the group scale (Fig. 4 caption),
//   pattern   min/max squared error against each pattern's first and last
//             centroid ("What carries the argument"; free parameters, Sec. 4.3),
//   quantise  onto the chosen pattern's 15 centroids, index 15 = the scale
//             element (free parameters),
//   codebook  the shortest of the pattern's 4 codebooks ("What carries the argument"),
//   pack      codewords into the 512-bit block, excess clipped (circularity
//             check, Sec. 3.2 step 9),
//   pad       spare bits filled with the largest remaining outliers, 15 bits
//             each, at most 16 (free parameters: "Number of padded outlier slots").
//
// Every fp32 operation is an explicitly rounded intrinsic (__fmul_rn, __fadd_rn,
// __fsub_rn, __fdiv_rn, __frcp_rn) so none is fused.  Tables are read through
// the read-only data cache (all lanes of a warp read the same pattern row), so
// a launch of a few thousand groups pays no per-CTA table staging.
#include "ecco_internal.cuh"

namespace ecco {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kEncWarps = 8;  // warps per CTA

struct Counters {  // warp-uniform
    uint32_t groups, zero, clipped, padded, records, nonfinite;
    unsigned long long bits;
};

__device__ __forceinline__ uint32_t pick4(uint32_t a, uint32_t b, uint32_t c, uint32_t d, int j)
{
    uint32_t lo = (j & 1) ? b : a;
    uint32_t hi = (j & 1) ? d : c;
    return (j & 2) ? hi : lo;
}

// Encodes the group at `src` into the block at `dst`.  All 32 lanes call it.
__device__ __forceinline__ void encode_group(const DevTables* __restrict__ tb, uint32_t* buf, float S_t,
                                             float2 endA, float2 endB, const uint16_t* src, uint8_t* dst,
                                             int lane, Counters& cnt)
{
    // ---- load 4 values (8 bytes per lane, 256 contiguous bytes per warp)
    uint2 raw = __ldg(reinterpret_cast<const uint2*>(src) + lane);
    uint32_t b0 = raw.x & 0xffffu, b1 = raw.x >> 16, b2 = raw.y & 0xffffu, b3 = raw.y >> 16;
    const int i0 = 4 * lane;

    // ---- first index of the largest magnitude: key = |x| << 7 | (127 - i)
    auto keyof = [&](uint32_t v, int i) { return ((v & 0x7fffu) << 7) | (uint32_t)(127 - i); };
    uint32_t key = max(max(keyof(b0, i0), keyof(b1, i0 + 1)), max(keyof(b2, i0 + 2), keyof(b3, i0 + 3)));
    key = __reduce_max_sync(kFull, key);
    if ((key >> 7) >= 0x7f80u) {  // a NaN or Inf in the group: encode it as +0 and recount
        int nf = 0;
        if ((b0 & 0x7f80u) == 0x7f80u) { b0 = 0; ++nf; }
        if ((b1 & 0x7f80u) == 0x7f80u) { b1 = 0; ++nf; }
        if ((b2 & 0x7f80u) == 0x7f80u) { b2 = 0; ++nf; }
        if ((b3 & 0x7f80u) == 0x7f80u) { b3 = 0; ++nf; }
        cnt.nonfinite += __reduce_add_sync(kFull, (uint32_t)nf);
        key = max(max(keyof(b0, i0), keyof(b1, i0 + 1)), max(keyof(b2, i0 + 2), keyof(b3, i0 + 3)));
        key = __reduce_max_sync(kFull, key);
    }
    const int m = 127 - (int)(key & 127u);
    const int mlane = m >> 2, mj = m & 3;
    const uint32_t xm_bits = __shfl_sync(kFull, pick4(b0, b1, b2, b3, mj), mlane);

    // ---- group scale: E4M3(x_m / S_t), round-half-even, saturating
    const float r = __fdiv_rn(bf16_bits_to_f32(xm_bits), S_t);
    const uint32_t code = (uint32_t)__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E4M3);
    const float fp8v = e4m3_to_f32(code);
    cnt.groups += 1;
    if (fp8v == 0.0f) {
        if (lane < 16) reinterpret_cast<uint32_t*>(dst)[lane] = 0u;
        cnt.zero += 1;
        return;
    }
    const float s = __fmul_rn(S_t, fp8v);
    const float inv = __frcp_rn(s);  // correctly rounded 1/s

    // ---- normalise; min / max over i != m (the scale element's slot takes the
    // value of a neighbour from the same lane, which leaves both extremes alone)
    float u0 = __fmul_rn(bf16_bits_to_f32(b0), inv), u1 = __fmul_rn(bf16_bits_to_f32(b1), inv);
    float u2 = __fmul_rn(bf16_bits_to_f32(b2), inv), u3 = __fmul_rn(bf16_bits_to_f32(b3), inv);
    float e0 = u0, e1 = u1, e2 = u2, e3 = u3;
    if (lane == mlane) {
        if (mj == 0) e0 = u1;
        if (mj == 1) e1 = u0;
        if (mj == 2) e2 = u3;
        if (mj == 3) e3 = u2;
    }
    const float umin = warp_min_f32(fminf(fminf(e0, e1), fminf(e2, e3)));
    const float umax = warp_max_f32(fmaxf(fmaxf(e0, e1), fmaxf(e2, e3)));

    // ---- pattern: lane holds patterns lane and lane + 32
    float d0 = __fsub_rn(umin, endA.x), d1 = __fsub_rn(umax, endA.y);
    const float ea = __fadd_rn(__fmul_rn(d0, d0), __fmul_rn(d1, d1));
    d0 = __fsub_rn(umin, endB.x);
    d1 = __fsub_rn(umax, endB.y);
    const float eb = __fadd_rn(__fmul_rn(d0, d0), __fmul_rn(d1, d1));
    const bool takeB = eb < ea;
    const uint32_t ebits = __float_as_uint(takeB ? eb : ea);  // e >= +0: bit order is value order
    const uint32_t emin = __reduce_min_sync(kFull, ebits);
    const int p = (int)__reduce_min_sync(kFull, ebits == emin ? (uint32_t)lane + (takeB ? 32u : 0u) : 64u);

    // ---- quantise: number of thresholds strictly below u (branchless search)
    const float* T = tb->T16[p];
    const float t7 = __ldg(T + 7);
    auto quant = [&](float v) {
        int idx = (t7 < v) ? 8 : 0;
        idx += (__ldg(T + idx + 3) < v) ? 4 : 0;
        idx += (__ldg(T + idx + 1) < v) ? 2 : 0;
        idx += (__ldg(T + idx) < v) ? 1 : 0;
        return (uint32_t)idx;
    };
    uint32_t s0 = quant(u0), s1 = quant(u1), s2 = quant(u2), s3 = quant(u3);
    if (lane == mlane) {
        if (mj == 0) s0 = 15;
        if (mj == 1) s1 = 15;
        if (mj == 2) s2 = 15;
        if (mj == 3) s3 = 15;
    }

    // ---- codebook: total length per codebook (4 byte lanes), shortest wins
    const uint32_t* L4 = tb->lens4[p];
    const uint32_t acc = __ldg(L4 + s0) + __ldg(L4 + s1) + __ldg(L4 + s2) + __ldg(L4 + s3);
    const uint32_t lo = __reduce_add_sync(kFull, acc & 0x00ff00ffu);         // h = 0, 2
    const uint32_t hi = __reduce_add_sync(kFull, (acc >> 8) & 0x00ff00ffu);  // h = 1, 3
    int h = 0, L = (int)(lo & 0xffffu);
    if ((int)(hi & 0xffffu) < L) { L = (int)(hi & 0xffffu); h = 1; }
    if ((int)(lo >> 16) < L) { L = (int)(lo >> 16); h = 2; }
    if ((int)(hi >> 16) < L) { L = (int)(hi >> 16); h = 3; }

    // ---- this lane's 4 codewords, concatenated in stream order (<= 32 bits)
    const uint32_t* CW = tb->code[p][h];
    const uint32_t c0 = __ldg(CW + s0), c1 = __ldg(CW + s1), c2 = __ldg(CW + s2), c3 = __ldg(CW + s3);
    const int l0 = (int)(c0 >> 8), l1 = (int)(c1 >> 8), l2 = (int)(c2 >> 8), l3 = (int)(c3 >> 8);
    uint32_t chunk = (c0 & 0xffu) | ((c1 & 0xffu) << l0);
    chunk |= (c2 & 0xffu) << (l0 + l1);
    chunk |= (c3 & 0xffu) << (l0 + l1 + l2);
    const int clen = l0 + l1 + l2 + l3;
    int off = clen;  // inclusive scan of chunk lengths
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        int t = __shfl_up_sync(kFull, off, d);
        if (lane >= d) off += t;
    }
    off -= clen;

    // ---- OR the chunks into the block; bits at or past 512 are dropped (clip)
    const int bpos = kHdrBits + off;
    const int w = bpos >> 5, sh = bpos & 31;
    if (w < 16) atomicOr(&buf[w], chunk << sh);
    if (sh != 0 && sh + clen > 32 && w + 1 < 16) atomicOr(&buf[w + 1], chunk >> (32 - sh));
    if (lane == 0) atomicOr(&buf[0], code | ((uint32_t)p << 8) | ((uint32_t)h << 14));

    // ---- outlier records in the spare bits of an unclipped block
    if (L <= kPayloadBits) {
        const int n = min(kMaxRec, (kPayloadBits - L) / kRecBits);
        if (n > 0) {
            // lane-local candidates, largest first (the scale element excluded)
            uint32_t k0 = keyof(b0, i0) + 1u, k1 = keyof(b1, i0 + 1) + 1u;
            uint32_t k2 = keyof(b2, i0 + 2) + 1u, k3 = keyof(b3, i0 + 3) + 1u;
            if (lane == mlane) {
                if (mj == 0) k0 = 0;
                if (mj == 1) k1 = 0;
                if (mj == 2) k2 = 0;
                if (mj == 3) k3 = 0;
            }
            // q for each of the lane's values: clamp(rint(u * 127), -127, 127)
            auto qof = [](float u) {
                float v = rintf(__fmul_rn(u, 127.0f));
                return (uint32_t)(int)fminf(fmaxf(v, -127.0f), 127.0f) & 0xffu;
            };
            const uint32_t rec0 = (uint32_t)i0 | (qof(u0) << 7), rec1 = (uint32_t)(i0 + 1) | (qof(u1) << 7);
            const uint32_t rec2 = (uint32_t)(i0 + 2) | (qof(u2) << 7), rec3 = (uint32_t)(i0 + 3) | (qof(u3) << 7);
            int at = kHdrBits + L;
            for (int k = 0; k < n; ++k, at += kRecBits) {
                uint32_t mine = max(max(k0, k1), max(k2, k3));
                uint32_t best = __reduce_max_sync(kFull, mine);
                if (mine == best) {  // exactly one lane: keys are unique
                    uint32_t rec;
                    if (best == k0) { rec = rec0; k0 = 0; }
                    else if (best == k1) { rec = rec1; k1 = 0; }
                    else if (best == k2) { rec = rec2; k2 = 0; }
                    else { rec = rec3; k3 = 0; }
                    const int ww = at >> 5, ss = at & 31;
                    atomicOr(&buf[ww], rec << ss);
                    if (ss > 32 - kRecBits) atomicOr(&buf[ww + 1], rec >> (32 - ss));
                }
            }
            cnt.records += n;
            cnt.padded += 1;
        }
        cnt.bits += L;
    } else {
        cnt.clipped += 1;
        cnt.bits += kPayloadBits;
    }

    __syncwarp();
    if (lane < 16) {
        reinterpret_cast<uint32_t*>(dst)[lane] = buf[lane];
        buf[lane] = 0u;
    }
    __syncwarp();
}

__global__ void __launch_bounds__(kEncWarps * 32)
    encode_kernel(const DevTables* __restrict__ tb, const uint16_t* __restrict__ x, ecco_desc d,
                  uint8_t* __restrict__ out, ecco_stats* __restrict__ stats, GridWalk walk)
{
    __shared__ uint32_t sbuf[kEncWarps][20];  // 16 block words + spill, per warp
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (lane < 20) sbuf[warp][lane] = 0u;
    const float2 endA = __ldg(&tb->ends[lane]);
    const float2 endB = __ldg(&tb->ends[lane + 32]);
    const float S_t = __ldg(&tb->S_t);
    __syncwarp();

    Counters cnt = {0, 0, 0, 0, 0, 0, 0ull};
    const int64_t gpr = d.groups_per_row;
    int64_t item = (int64_t)blockIdx.x * kEncWarps + warp;
    int64_t r = item / gpr, g = item - r * gpr;
    const int64_t step = (int64_t)gridDim.x * kEncWarps;
    for (; item < walk.total; item += step) {
        const uint16_t* src = x + (d.src_offset + r * d.src_row_stride + g) * kG;
        uint8_t* dst = out + (d.dst_offset + r * d.dst_row_stride + g) * ECCO_BLOCK_BYTES;
        encode_group(tb, sbuf[warp], S_t, endA, endB, src, dst, lane, cnt);
        g += walk.stride_g;
        r += walk.stride_r;
        if (g >= gpr) {
            g -= gpr;
            r += 1;
        }
    }
    if (stats && lane == 0 && cnt.groups) {  // counters are warp-uniform
        atomicAdd(&stats->n_groups, (unsigned long long)cnt.groups);
        if (cnt.zero) atomicAdd(&stats->n_zero, (unsigned long long)cnt.zero);
        if (cnt.clipped) atomicAdd(&stats->n_clipped, (unsigned long long)cnt.clipped);
        if (cnt.padded) atomicAdd(&stats->n_padded, (unsigned long long)cnt.padded);
        if (cnt.records) atomicAdd(&stats->n_records, (unsigned long long)cnt.records);
        if (cnt.nonfinite) atomicAdd(&stats->n_nonfinite, (unsigned long long)cnt.nonfinite);
        if (cnt.bits) atomicAdd(&stats->payload_bits, cnt.bits);
    }
}

}  // namespace

cudaError_t launch_encode(const ecco_tables* t, const uint16_t* x, const ecco_desc& d,
                          uint8_t* blocks, ecco_stats* stats, cudaStream_t s)
{
    const int64_t total = d.rows * d.groups_per_row;
    const int per_cta = kEncWarps;
    int64_t want = (total + per_cta - 1) / per_cta;
    int64_t cap = (int64_t)device_sm_count() * 8;  // resident warps to hide latency
    int grid = (int)(want < cap ? want : cap);
    GridWalk walk;
    walk.total = total;
    int64_t stride = (int64_t)grid * per_cta;
    walk.stride_r = stride / d.groups_per_row;
    walk.stride_g = stride % d.groups_per_row;
    encode_kernel<<<grid, kEncWarps * 32, 0, s>>>(t->d, x, d, blocks, stats, walk);
    return cudaGetLastError();
}

}  // namespace ecco
