// Decoder: one thread per 512-bit block.
//
// The review page's decompressor ("Ecco: Improving Memory Bandwidth and
// Capacity for LLMs via Entropy-aware Cache Compression", Fig. 8 caption and
// referee comment 1) is a 64-way hardware decoder that speculates at every bit
// offset to beat the serial dependency of one variable-length stream.  A
// B200 has millions of independent blocks in flight instead, so here every
// thread walks one block's stream serially and parallelism comes from the
// blocks: the serial chain (one shared-memory table lookup per symbol) is
// hidden by 32 resident warps per SM, and no work is spent on offsets that
// turn out to be wrong.
//
// Per block: parse the header (scale code, pattern, codebook), form the 16
// output values bf16(s * C[p][j]) as register byte planes, decode the stream
// 8 symbols at a time (ecco_block.cuh), write each 16 decoded values with one
// 32-byte store, then apply the outlier records of an unclipped stream.
#include "ecco_block.cuh"

namespace ecco {
namespace {

constexpr int kDecThreads = 1024;
constexpr int kWordStride = kDecThreads;  // word k of thread t at k * stride + t: conflict-free

constexpr size_t kDecSmemLut = sizeof(((DevTables*)0)->lut);  // 65536
constexpr size_t kDecSmemCt = sizeof(((DevTables*)0)->Ct);    // 4096
constexpr size_t kDecSmemWords = 16 * kWordStride * 4;
constexpr size_t kDecSmem = kDecSmemLut + kDecSmemCt + kDecSmemWords;

// WIDE: 32-byte stores (output 32-byte aligned), else 16-byte stores.
template <bool WIDE>
__device__ __forceinline__ void store16(uint16_t* dst, const uint32_t a[4], const uint32_t b[4])
{
    if (WIDE) {
        stg256(dst, a, b);
    } else {
        *reinterpret_cast<uint4*>(dst) = make_uint4(a[0], a[1], a[2], a[3]);
        *reinterpret_cast<uint4*>(dst + 8) = make_uint4(b[0], b[1], b[2], b[3]);
    }
}

template <bool WIDE>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_kernel(const DevTables* __restrict__ tb, const uint8_t* __restrict__ blocks, ecco_desc d,
                  uint16_t* __restrict__ y, GridWalk walk)
{
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t* s_lut = smem;
    float* s_Ct = reinterpret_cast<float*>(smem + kDecSmemLut);
    uint32_t* s_w = reinterpret_cast<uint32_t*>(smem + kDecSmemLut + kDecSmemCt);
    const int tid = threadIdx.x;
    {
        const uint4* a = reinterpret_cast<const uint4*>(&tb->lut[0][0]);
        uint4* b = reinterpret_cast<uint4*>(s_lut);
        for (int i = tid; i < (int)(kDecSmemLut / 16); i += kDecThreads) b[i] = a[i];
        const uint4* c = reinterpret_cast<const uint4*>(&tb->Ct[0][0]);
        uint4* e = reinterpret_cast<uint4*>(s_Ct);
        for (int i = tid; i < (int)(kDecSmemCt / 16); i += kDecThreads) e[i] = c[i];
    }
    const float S_t = tb->S_t;
    __syncthreads();

    uint32_t* ws = s_w + tid;
    const int64_t gpr = d.groups_per_row;
    // Item order: consecutive lanes take consecutive blocks; the warps of a
    // round are spread over all CTAs first, so a partial last round is shared
    // by every SM instead of loading the first few.
    int64_t item = ((int64_t)(tid >> 5) * gridDim.x + blockIdx.x) * 32 + (tid & 31);
    int64_t r = item / gpr, g = item - r * gpr;
    for (; item < walk.total; item += (int64_t)gridDim.x * kDecThreads) {
        const uint8_t* src = blocks + (d.src_offset + r * d.src_row_stride + g) * ECCO_BLOCK_BYTES;
        uint16_t* dst = y + (d.dst_offset + r * d.dst_row_stride + g) * kG;
        g += walk.stride_g;
        r += walk.stride_r;
        if (g >= gpr) {
            g -= gpr;
            r += 1;
        }

        uint4 q0 = ldg_nc_v4(src), q1 = ldg_nc_v4(src + 16), q2 = ldg_nc_v4(src + 32),
              q3 = ldg_nc_v4(src + 48);
        const uint32_t code = q0.x & 0xffu;
        if (scale_code_is_null(code)) {
            const uint32_t z[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int k = 0; k < 8; ++k) store16<WIDE>(dst + 16 * k, z, z);
            continue;
        }
        stage_words(ws, kWordStride, q0, q1, q2, q3);
        const int p = (int)((q0.x >> 8) & 63u);
        const uint8_t* lut = s_lut + ((q0.x >> 8) & 255u) * 256;  // table h * 64 + p
        const float s = __fmul_rn(S_t, e4m3_to_f32(code));
        const ValuePlanes vp = make_planes(s, s_Ct, p);

        Stream st{q0.x, q0.y, kHdrBits, 2, kPayloadBits};
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {  // 8 x 16 symbols, one 32-byte store each
            uint32_t wa[4], wb[4];
            chunk_values(st, lut, ws, kWordStride, vp, wa);
            chunk_values(st, lut, ws, kWordStride, vp, wb);
            store16<WIDE>(dst + 16 * c, wa, wb);
        }

        if (st.room >= 0) {  // unclipped: outlier records follow the codewords
            const int n = min(kMaxRec, st.room / kRecBits);
            int at = kBlockBits - st.room;
            for (int k = 0; k < n; ++k, at += kRecBits) {
                uint32_t rec = read_record(ws, kWordStride, at);
                int i = (int)(rec & 127u);
                int qv = (int)(int8_t)(uint8_t)(rec >> 7);
                float o = __fdiv_rn((float)qv, 127.0f);
                dst[i] = (uint16_t)f32_to_bf16_bits(__fmul_rn(s, o));
            }
        }
    }
}

}  // namespace

cudaError_t launch_decode(const ecco_tables* t, const uint8_t* blocks, const ecco_desc& d,
                          uint16_t* y, cudaStream_t s)
{
    static int configured_dev = -1;
    int dev = t->device;
    if (configured_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kDecSmem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kDecSmem);
        if (e != cudaSuccess) return e;
        configured_dev = dev;
    }
    const int64_t total = d.rows * d.groups_per_row;
    int64_t want = (total + kDecThreads - 1) / kDecThreads;
    int64_t cap = device_sm_count();
    int grid = (int)(want < cap ? want : cap);
    GridWalk walk;
    walk.total = total;
    int64_t stride = (int64_t)grid * kDecThreads;
    walk.stride_r = stride / d.groups_per_row;
    walk.stride_g = stride % d.groups_per_row;
    if ((reinterpret_cast<uintptr_t>(y) & 31u) == 0)
        decode_kernel<true><<<grid, kDecThreads, kDecSmem, s>>>(t->d, blocks, d, y, walk);
    else
        decode_kernel<false><<<grid, kDecThreads, kDecSmem, s>>>(t->d, blocks, d, y, walk);
    return cudaGetLastError();
}

}  // namespace ecco
