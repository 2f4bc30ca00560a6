// Decode-phase attention read straight from the compressed KV cache.
//
// The review page ("Ecco: Improving Memory Bandwidth and Capacity for LLMs via
// Entropy-aware Cache Compression", "If this is right" and the Fig. 11
// caption) places Ecco's gains in the memory-bound decode phase at long
// sequence lengths: the KV cache is read in compressed form and decompressed
// on the way to the SMs.  Here the attention kernel itself decodes the K and
// V blocks, so the bf16 cache is never written to or read from memory.
//
// For each (batch b, KV head h) the sequence is cut into splits of 512 tokens
// (flash-decoding).  One CTA of 512 threads owns a split; thread t owns token
// split * 512 + t:
//   K pass  decode the token's K block and form the G query heads' scores
//           q . k~ * scale on the fly (q broadcast from shared memory);
//           outlier records correct the dot products by (new - old) * q.
//   softmax CTA-wide max and exp per query head.
//   V pass  decode the token's V block; every 32 dimensions the warp
//           transposes its 32 tokens through shared memory so that each lane
//           accumulates p . v~ for one dimension, then adds it to the CTA's
//           [G][128] accumulator (shared-memory atomics); records add
//           p * (new - old) to the same accumulator.
// Partial (max, sum, p.V) of every split go to a caller-owned workspace; a
// second kernel merges the splits with the usual log-sum-exp rescaling.
#include "ecco_block.cuh"

namespace ecco {
namespace {

constexpr int kAtThreads = 512;
constexpr int kAtWarps = kAtThreads / 32;
constexpr int kAtStride = kAtThreads;
constexpr int kStageRow = 20;  // words per staged token row (32 bf16 + pad: conflict-free)

struct AttnArgs {
    const DevTables* ktb;
    const DevTables* vtb;
    const uint8_t* kblk;
    const uint8_t* vblk;
    int64_t s_cap;
    int H, G, S, splits;
    const uint16_t* q;
    float scale;
    float* ws;  // [B][H*G][splits][130]: 128 partial p.V, then max, sum
};

template <int G>
constexpr size_t attn_smem()
{
    return 65536 + 4096                           // decode tables, centroids
           + (size_t)16 * kAtStride * 4           // stream words
           + (size_t)kAtWarps * 32 * kStageRow * 4  // per-warp V staging
           + (size_t)G * 128 * 4                  // q
           + (size_t)G * kAtThreads * 4           // scores / probabilities
           + (size_t)kAtWarps * G * 4 * 2         // reductions
           + (size_t)G * 128 * 4;                 // p.V accumulator
}

// Loads one block, returns its scale (0 for a null scale or a token past the end).
__device__ __forceinline__ float load_block(const uint8_t* src, bool ok, uint4& q0, uint4& q1, uint4& q2,
                                            uint4& q3, float S_t)
{
    q0 = q1 = q2 = q3 = make_uint4(0, 0, 0, 0);
    if (ok) {
        q0 = ldg_nc_v4(src);
        q1 = ldg_nc_v4(src + 16);
        q2 = ldg_nc_v4(src + 32);
        q3 = ldg_nc_v4(src + 48);
    }
    const uint32_t code = q0.x & 0xffu;
    return (ok && !scale_code_is_null(code)) ? __fmul_rn(S_t, e4m3_to_f32(code)) : 0.0f;
}

__device__ __forceinline__ float value_of(const ValuePlanes& vp, uint32_t sym)
{
    uint32_t ow = (sym < 8) ? ((sym < 4) ? vp.lo[0] : vp.lo[1]) : ((sym < 12) ? vp.lo[2] : vp.lo[3]);
    uint32_t oh = (sym < 8) ? ((sym < 4) ? vp.hi[0] : vp.hi[1]) : ((sym < 12) ? vp.hi[2] : vp.hi[3]);
    uint32_t sh = 8 * (sym & 3);
    return __uint_as_float((((ow >> sh) & 0xffu) | (((oh >> sh) & 0xffu) << 8)) << 16);
}

// Calls f(i, new_value - old_value) for every outlier record of an unclipped
// block whose value is final (the last record of an element wins).
template <class F>
__device__ __forceinline__ void for_records(const Stream& st, const uint32_t* ws, int stride, float s,
                                            const ValuePlanes& vp, const uint32_t nib[16], F f)
{
    if (s == 0.0f || st.room < 0) return;
    const int n = min(kMaxRec, st.room / kRecBits);
    const int at0 = kBlockBits - st.room;
    for (int k = n - 1; k >= 0; --k) {
        const uint32_t rec = read_record(ws, stride, at0 + k * kRecBits);
        const int i = (int)(rec & 127u);
        bool later = false;
        for (int k2 = k + 1; k2 < n; ++k2)
            later = later || ((int)(read_record(ws, stride, at0 + k2 * kRecBits) & 127u) == i);
        if (later) continue;
        const int qv = (int)(int8_t)(uint8_t)(rec >> 7);
        const float nv = bf16_bits_to_f32(f32_to_bf16_bits(__fmul_rn(s, __fdiv_rn((float)qv, 127.0f))));
        uint32_t word = nib[0];
#pragma unroll
        for (int c = 1; c < 16; ++c) word = ((i >> 3) == c) ? nib[c] : word;
        const float ov = value_of(vp, (word >> (4 * (i & 7))) & 15u);
        f(i, nv - ov);
    }
}

template <int G>
__global__ void __launch_bounds__(kAtThreads, 1) attn_split_kernel(const __grid_constant__ AttnArgs A)
{
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t* s_lut = smem;
    float* s_Ct = reinterpret_cast<float*>(smem + 65536);
    uint32_t* s_w = reinterpret_cast<uint32_t*>(smem + 65536 + 4096);
    uint32_t* s_stage = s_w + 16 * kAtStride;
    float* s_q = reinterpret_cast<float*>(s_stage + kAtWarps * 32 * kStageRow);
    float* s_p = s_q + G * 128;
    float* s_red = s_p + G * kAtThreads;
    float* s_acc = s_red + kAtWarps * G * 2;  // [G][128]: p.V of the split (shared atomics)

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = blockIdx.x, bh = blockIdx.y;
    const int b = bh / A.H, h = bh - b * A.H;
    const int Hq = A.H * G;
    const int s_tok = split * kAtThreads + tid;
    const bool have = s_tok < A.S;
    const int64_t blk = (int64_t)bh * A.s_cap + s_tok;

    // q of the group's heads (fp32), corrections cleared
    for (int i = tid; i < G * 128; i += kAtThreads) {
        const int g = i >> 7, d = i & 127;
        s_q[i] = bf16_bits_to_f32(A.q[((int64_t)b * Hq + h * G + g) * 128 + d]);
        s_acc[i] = 0.0f;
    }
    stage_tables<kAtThreads>(A.ktb, s_lut, s_Ct, tid);
    __syncthreads();

    uint32_t* ws = s_w + tid;
    uint32_t nib[16];

    // ---------------- K pass: scores
    float dot[G];
#pragma unroll
    for (int g = 0; g < G; ++g) dot[g] = 0.0f;
    {
        uint4 q0, q1, q2, q3;
        const float s = load_block(A.kblk + blk * ECCO_BLOCK_BYTES, have, q0, q1, q2, q3, A.ktb->S_t);
        stage_words(ws, kAtStride, q0, q1, q2, q3);
        const ValuePlanes vp = make_planes(s, s_Ct, (int)((q0.x >> 8) & 63u));
        const uint8_t* lut = s_lut + ((q0.x >> 8) & 255u) * 256;
        Stream st{q0.x, q0.y, kHdrBits, 2, kPayloadBits};
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            uint32_t w[4];
            nib[c] = chunk_values(st, lut, ws, kAtStride, vp, w);
            float v[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                v[2 * j] = __uint_as_float(w[j] << 16);
                v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float4 qa = *reinterpret_cast<const float4*>(s_q + g * 128 + 8 * c);
                const float4 qb = *reinterpret_cast<const float4*>(s_q + g * 128 + 8 * c + 4);
                dot[g] = fmaf(v[0], qa.x, dot[g]);
                dot[g] = fmaf(v[1], qa.y, dot[g]);
                dot[g] = fmaf(v[2], qa.z, dot[g]);
                dot[g] = fmaf(v[3], qa.w, dot[g]);
                dot[g] = fmaf(v[4], qb.x, dot[g]);
                dot[g] = fmaf(v[5], qb.y, dot[g]);
                dot[g] = fmaf(v[6], qb.z, dot[g]);
                dot[g] = fmaf(v[7], qb.w, dot[g]);
            }
        }
        for_records(st, ws, kAtStride, s, vp, nib, [&](int i, float dv) {
#pragma unroll
            for (int g = 0; g < G; ++g) dot[g] = fmaf(dv, s_q[g * 128 + i], dot[g]);
        });
    }

    // ---------------- softmax over this split's tokens
    float m[G], l[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const float sc = have ? dot[g] * A.scale : -INFINITY;
        float mx = sc;
#pragma unroll
        for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) s_red[warp * G + g] = mx;
        dot[g] = sc;
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float mx = -INFINITY;
        for (int w = 0; w < kAtWarps; ++w) mx = fmaxf(mx, s_red[w * G + g]);
        m[g] = mx;
        const float p = have ? expf(dot[g] - mx) : 0.0f;
        s_p[g * kAtThreads + tid] = p;
        float sum = p;
#pragma unroll
        for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) s_red[kAtWarps * G + warp * G + g] = sum;
    }
    __syncthreads();  // also: K tables no longer read
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float sum = 0.0f;
        for (int w = 0; w < kAtWarps; ++w) sum += s_red[kAtWarps * G + w * G + g];
        l[g] = sum;
    }
    stage_tables<kAtThreads>(A.vtb, s_lut, s_Ct, tid);
    __syncthreads();

    // ---------------- V pass
    {
        uint4 q0, q1, q2, q3;
        const float s = load_block(A.vblk + blk * ECCO_BLOCK_BYTES, have, q0, q1, q2, q3, A.vtb->S_t);
        stage_words(ws, kAtStride, q0, q1, q2, q3);
        const ValuePlanes vp = make_planes(s, s_Ct, (int)((q0.x >> 8) & 63u));
        const uint8_t* lut = s_lut + ((q0.x >> 8) & 255u) * 256;
        Stream st{q0.x, q0.y, kHdrBits, 2, kPayloadBits};
        uint32_t* stage = s_stage + warp * 32 * kStageRow;
        const float* pw = s_p + warp * 32;  // probabilities of this warp's 32 tokens
#pragma unroll
        for (int grp = 0; grp < 4; ++grp) {
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                uint32_t w[4];
                nib[grp * 4 + c4] = chunk_values(st, lut, ws, kAtStride, vp, w);
                *reinterpret_cast<uint4*>(stage + lane * kStageRow + 4 * c4) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            __syncwarp();
            // lane = dimension 32 * grp + lane; the warp's 32 tokens in turn
            const uint16_t* col = reinterpret_cast<const uint16_t*>(stage) + lane;
            float acc[G];
#pragma unroll
            for (int g = 0; g < G; ++g) acc[g] = 0.0f;
#pragma unroll 2
            for (int t = 0; t < 32; t += 4) {
                float v[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) v[k] = bf16_bits_to_f32(col[(t + k) * 2 * kStageRow]);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float4 p4 = *reinterpret_cast<const float4*>(pw + g * kAtThreads + t);
                    acc[g] = fmaf(p4.x, v[0], acc[g]);
                    acc[g] = fmaf(p4.y, v[1], acc[g]);
                    acc[g] = fmaf(p4.z, v[2], acc[g]);
                    acc[g] = fmaf(p4.w, v[3], acc[g]);
                }
            }
#pragma unroll
            for (int g = 0; g < G; ++g) atomicAdd(&s_acc[g * 128 + grp * 32 + lane], acc[g]);
            __syncwarp();
        }
        for_records(st, ws, kAtStride, s, vp, nib, [&](int i, float dv) {
#pragma unroll
            for (int g = 0; g < G; ++g) atomicAdd(&s_acc[g * 128 + i], s_p[g * kAtThreads + tid] * dv);
        });
    }
    __syncthreads();

    // ---------------- this split's partial result
    float* out = A.ws + ((int64_t)b * Hq + h * G) * A.splits * 130;
    for (int i = tid; i < G * 128; i += kAtThreads) {
        const int g = i >> 7, d = i & 127;
        out[((int64_t)g * A.splits + split) * 130 + d] = s_acc[i];
    }
    if (tid == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            out[((int64_t)g * A.splits + split) * 130 + 128] = m[g];
            out[((int64_t)g * A.splits + split) * 130 + 129] = l[g];
        }
    }
}

// One CTA of 128 threads per (batch, query head): merge the splits.
__global__ void __launch_bounds__(128) attn_merge_kernel(const float* __restrict__ ws, int splits,
                                                          float* __restrict__ out)
{
    const int bq = blockIdx.x, d = threadIdx.x;
    const float* part = ws + (int64_t)bq * splits * 130;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, part[s * 130 + 128]);
    float L = 0.0f, acc = 0.0f;
    for (int s = 0; s < splits; ++s) {
        const float w = expf(part[s * 130 + 128] - M);
        L = fmaf(part[s * 130 + 129], w, L);
        acc = fmaf(part[s * 130 + d], w, acc);
    }
    out[(int64_t)bq * 128 + d] = acc / L;
}

template <int G>
cudaError_t run_attn(const AttnArgs& A, int B, cudaStream_t s, float* out)
{
    static int configured = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured != dev) {
        cudaError_t e = cudaFuncSetAttribute(attn_split_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)attn_smem<G>());
        if (e != cudaSuccess) return e;
        configured = dev;
    }
    dim3 grid((unsigned)A.splits, (unsigned)(B * A.H));
    attn_split_kernel<G><<<grid, kAtThreads, attn_smem<G>(), s>>>(A);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_merge_kernel<<<B * A.H * G, 128, 0, s>>>(A.ws, A.splits, out);
    return cudaGetLastError();
}

}  // namespace

int attention_splits(int seq_len) { return (seq_len + kAtThreads - 1) / kAtThreads; }

cudaError_t launch_attention(const ecco_tables* kt, const ecco_tables* vt, const uint8_t* kblk,
                             const uint8_t* vblk, int64_t s_cap, int B, int H, int G, int S,
                             const uint16_t* q, float scale, float* out, float* ws, cudaStream_t s)
{
    AttnArgs A{kt->d, vt->d, kblk, vblk, s_cap, H, G, S, attention_splits(S), q, scale, ws};
    switch (G) {
        case 1: return run_attn<1>(A, B, s, out);
        case 2: return run_attn<2>(A, B, s, out);
        case 3: return run_attn<3>(A, B, s, out);
        case 4: return run_attn<4>(A, B, s, out);
        case 5: return run_attn<5>(A, B, s, out);
        case 6: return run_attn<6>(A, B, s, out);
        case 7: return run_attn<7>(A, B, s, out);
        case 8: return run_attn<8>(A, B, s, out);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ecco
