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
// Arithmetic: every fp32 operation is an explicitly rounded intrinsic
// (__fmul_rn, __fadd_rn, __fsub_rn, __fdiv_rn, __frcp_rn) so none is fused.
#include "ecco_internal.cuh"

namespace ecco {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kEncWarps = 8;  // warps per CTA

struct EncShared {
    float T[kNPat][16];
    uint32_t lens4[kNPat][16];
    uint32_t code[kNPat][kNBook][16];
    uint32_t buf[kEncWarps][20];  // 16 block words + spill word, per warp
};

struct Counters {
    unsigned long long groups, zero, clipped, padded, records, nonfinite, bits;
};

__device__ __forceinline__ uint32_t sel4(const uint32_t v[4], int j)
{
    uint32_t r = v[0];
    r = (j == 1) ? v[1] : r;
    r = (j == 2) ? v[2] : r;
    r = (j == 3) ? v[3] : r;
    return r;
}

__device__ __forceinline__ float self4(const float v[4], int j)
{
    float r = v[0];
    r = (j == 1) ? v[1] : r;
    r = (j == 2) ? v[2] : r;
    r = (j == 3) ? v[3] : r;
    return r;
}

// Encodes the group at `src` into the block at `dst`.  All 32 lanes call it.
__device__ __forceinline__ void encode_group(const EncShared& sh, uint32_t* buf, float S_t,
                                             float2 endA, float2 endB, const uint16_t* src,
                                             uint8_t* dst, int lane, Counters& cnt)
{
    // ---- load 4 values (8 bytes per lane, 256 contiguous bytes per warp)
    uint2 raw = __ldg(reinterpret_cast<const uint2*>(src) + lane);
    uint32_t b[4] = {raw.x & 0xffffu, raw.x >> 16, raw.y & 0xffffu, raw.y >> 16};
    int nonfin = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        if ((b[j] & 0x7f80u) == 0x7f80u) {  // NaN / Inf -> +0
            b[j] = 0;
            nonfin++;
        }
    cnt.nonfinite += nonfin;

    // ---- first index of the largest magnitude: key = |x| << 7 | (127 - i)
    uint32_t key = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t k = ((b[j] & 0x7fffu) << 7) | (uint32_t)(127 - (4 * lane + j));
        key = max(key, k);
    }
    key = __reduce_max_sync(kFull, key);
    const int m = 127 - (int)(key & 127u);
    const int mlane = m >> 2, mj = m & 3;
    uint32_t xm_bits = __shfl_sync(kFull, sel4(b, mj), mlane);

    // ---- group scale: E4M3(x_m / S_t), round-half-even, saturating
    float xm = bf16_bits_to_f32(xm_bits);
    float r = __fdiv_rn(xm, S_t);
    uint32_t code = (uint32_t)__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E4M3);
    float fp8v = e4m3_to_f32(code);
    cnt.groups += 1;
    if (fp8v == 0.0f) {
        if (lane < 16) reinterpret_cast<uint32_t*>(dst)[lane] = 0u;
        cnt.zero += 1;
        return;
    }
    const float s = __fmul_rn(S_t, fp8v);
    const float inv = __frcp_rn(s);  // correctly rounded 1/s

    // ---- normalise; min / max over i != m
    float u[4];
    float lmin = INFINITY, lmax = -INFINITY;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        u[j] = __fmul_rn(bf16_bits_to_f32(b[j]), inv);
        if (4 * lane + j != m) {
            lmin = fminf(lmin, u[j]);
            lmax = fmaxf(lmax, u[j]);
        }
    }
    const float umin = warp_min_f32(lmin);
    const float umax = warp_max_f32(lmax);

    // ---- pattern: lane holds patterns lane and lane + 32
    float d0 = __fsub_rn(umin, endA.x), d1 = __fsub_rn(umax, endA.y);
    float ea = __fadd_rn(__fmul_rn(d0, d0), __fmul_rn(d1, d1));
    d0 = __fsub_rn(umin, endB.x);
    d1 = __fsub_rn(umax, endB.y);
    float eb = __fadd_rn(__fmul_rn(d0, d0), __fmul_rn(d1, d1));
    float e = ea;
    uint32_t pl = (uint32_t)lane;
    if (eb < ea) {
        e = eb;
        pl = (uint32_t)lane + 32u;
    }
    uint32_t ebits = __float_as_uint(e);  // e >= +0: bit order is value order
    uint32_t emin = __reduce_min_sync(kFull, ebits);
    const int p = (int)__reduce_min_sync(kFull, ebits == emin ? pl : 64u);

    // ---- quantise: count of thresholds strictly below u (branchless search)
    const float* T = sh.T[p];
    uint32_t sym[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float v = u[j];
        int idx = (T[7] < v) ? 8 : 0;
        idx += (T[idx + 3] < v) ? 4 : 0;
        idx += (T[idx + 1] < v) ? 2 : 0;
        idx += (T[idx] < v) ? 1 : 0;
        sym[j] = (4 * lane + j == m) ? 15u : (uint32_t)idx;
    }

    // ---- codebook: total length per codebook (4 byte lanes), shortest wins
    uint32_t acc = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) acc += sh.lens4[p][sym[j]];
    uint32_t lo = __reduce_add_sync(kFull, acc & 0x00ff00ffu);         // h = 0, 2
    uint32_t hi = __reduce_add_sync(kFull, (acc >> 8) & 0x00ff00ffu);  // h = 1, 3
    int Lh[4] = {(int)(lo & 0xffffu), (int)(hi & 0xffffu), (int)(lo >> 16), (int)(hi >> 16)};
    int h = 0, L = Lh[0];
#pragma unroll
    for (int k = 1; k < 4; ++k)
        if (Lh[k] < L) {
            L = Lh[k];
            h = k;
        }

    // ---- this lane's 4 codewords, concatenated in stream order (<= 32 bits)
    uint32_t chunk = 0;
    int clen = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t c = sh.code[p][h][sym[j]];
        chunk |= (c & 0xffu) << clen;
        clen += (int)((c >> 8) & 15u);
    }
    int off = clen;  // inclusive scan of chunk lengths
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        int t = __shfl_up_sync(kFull, off, d);
        if (lane >= d) off += t;
    }
    off -= clen;

    // ---- OR the chunks into the block; bits at or past 512 are dropped (clip)
    int bpos = kHdrBits + off;
    int w = bpos >> 5, sh_ = bpos & 31;
    if (w < 16) atomicOr(&buf[w], chunk << sh_);
    if (sh_ != 0 && sh_ + clen > 32 && w + 1 < 16) atomicOr(&buf[w + 1], chunk >> (32 - sh_));
    if (lane == 0) atomicOr(&buf[0], code | ((uint32_t)p << 8) | ((uint32_t)h << 14));

    // ---- outlier records in the spare bits of an unclipped block
    if (L <= kPayloadBits) {
        int n = min(kMaxRec, (kPayloadBits - L) / kRecBits);
        uint32_t taken = (lane == mlane) ? (1u << mj) : 0u;
        for (int k = 0; k < n; ++k) {
            uint32_t best = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t c = (((b[j] & 0x7fffu) << 7) | (uint32_t)(127 - (4 * lane + j))) + 1u;
                if (!((taken >> j) & 1u)) best = max(best, c);
            }
            best = __reduce_max_sync(kFull, best);
            int i = 127 - (int)((best - 1u) & 127u);
            int owner = i >> 2, ij = i & 3;
            int q = 0;
            if (lane == owner) {
                taken |= 1u << ij;
                float v = rintf(__fmul_rn(self4(u, ij), 127.0f));
                v = fminf(fmaxf(v, -127.0f), 127.0f);
                q = (int)v;
            }
            q = __shfl_sync(kFull, q, owner);
            if (lane == 0) {
                uint32_t rec = (uint32_t)i | (((uint32_t)q & 0xffu) << 7);
                int at = kHdrBits + L + kRecBits * k;
                int ww = at >> 5, ss = at & 31;
                atomicOr(&buf[ww], rec << ss);
                if (ss > 32 - kRecBits && ww + 1 < 16) atomicOr(&buf[ww + 1], rec >> (32 - ss));
            }
        }
        cnt.records += n;
        cnt.padded += (n > 0);
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
    __shared__ EncShared sh;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    {
        const uint4* src = reinterpret_cast<const uint4*>(&tb->T16[0][0]);
        uint4* dstT = reinterpret_cast<uint4*>(&sh.T[0][0]);
        for (int i = tid; i < (int)(sizeof(sh.T) / 16); i += blockDim.x) dstT[i] = src[i];
        const uint4* srcL = reinterpret_cast<const uint4*>(&tb->lens4[0][0]);
        uint4* dstL = reinterpret_cast<uint4*>(&sh.lens4[0][0]);
        for (int i = tid; i < (int)(sizeof(sh.lens4) / 16); i += blockDim.x) dstL[i] = srcL[i];
        const uint4* srcC = reinterpret_cast<const uint4*>(&tb->code[0][0][0]);
        uint4* dstC = reinterpret_cast<uint4*>(&sh.code[0][0][0]);
        for (int i = tid; i < (int)(sizeof(sh.code) / 16); i += blockDim.x) dstC[i] = srcC[i];
        for (int i = tid; i < kEncWarps * 20; i += blockDim.x) (&sh.buf[0][0])[i] = 0u;
    }
    const float2 endA = tb->ends[lane];
    const float2 endB = tb->ends[lane + 32];
    const float S_t = tb->S_t;
    __syncthreads();

    Counters cnt = {0, 0, 0, 0, 0, 0, 0};
    const int64_t gpr = d.groups_per_row;
    int64_t item = (int64_t)blockIdx.x * kEncWarps + warp;
    int64_t r = item / gpr, g = item - r * gpr;
    for (; item < walk.total; item += (int64_t)gridDim.x * kEncWarps) {
        const uint16_t* src = x + (d.src_offset + r * d.src_row_stride + g) * kG;
        uint8_t* dst = out + (d.dst_offset + r * d.dst_row_stride + g) * ECCO_BLOCK_BYTES;
        encode_group(sh, sh.buf[warp], S_t, endA, endB, src, dst, lane, cnt);
        g += walk.stride_g;
        r += walk.stride_r;
        if (g >= gpr) {
            g -= gpr;
            r += 1;
        }
    }
    if (stats && lane == 0) {  // counters are warp-uniform
        if (cnt.groups) atomicAdd(&stats->n_groups, cnt.groups);
        if (cnt.zero) atomicAdd(&stats->n_zero, cnt.zero);
        if (cnt.clipped) atomicAdd(&stats->n_clipped, cnt.clipped);
        if (cnt.padded) atomicAdd(&stats->n_padded, cnt.padded);
        if (cnt.records) atomicAdd(&stats->n_records, cnt.records);
        if (cnt.bits) atomicAdd(&stats->payload_bits, cnt.bits);
    }
    if (stats) {
        unsigned long long nf = cnt.nonfinite;
        for (int o = 16; o; o >>= 1) nf += __shfl_down_sync(kFull, nf, o);
        if (lane == 0 && nf) atomicAdd(&stats->n_nonfinite, nf);
    }
}

}  // namespace

cudaError_t launch_encode(const ecco_tables* t, const uint16_t* x, const ecco_desc& d,
                          uint8_t* blocks, ecco_stats* stats, cudaStream_t s)
{
    const int64_t total = d.rows * d.groups_per_row;
    const int per_cta = kEncWarps;
    int64_t want = (total + per_cta - 1) / per_cta;
    int64_t cap = (int64_t)device_sm_count() * 8;  // enough resident warps to hide latency
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
