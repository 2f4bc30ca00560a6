// Fused decode + matrix-vector product on CUDA cores (batch 1..4; larger
// batches go to the tensor-core kernel in ecco_gemm_tc.cu).
//
// y[b][r] = sum_k W~[r][k] * x[b][k], W~ the decoded matrix, never written to
// memory (the review page's figure list: "Normalized Memory Requests for a
// GEMM Kernel" -- compressed weights are what crosses the memory bus).
//
// Layout of the work: a warp owns 32 consecutive rows and walks a range of
// column groups in lockstep, so at every step all lanes need the same x[k]
// (a broadcast shared-memory read).  Each lane decodes its row's block
// serially (one lookup per symbol, as in the decoder) and multiplies every
// decoded bf16 value, exactly, in fp32 against the batch of x.  An outlier
// record replaces the value of its element, so its contribution is corrected
// by (new - old) * x, with the old symbol kept in shared memory.  Partial row
// sums of the column ranges are combined with fp32 atomics.
#include "ecco_block.cuh"

namespace ecco {
namespace {

constexpr int kGvThreads = 512;
constexpr int kGvWarps = kGvThreads / 32;
constexpr int kGvColGroups = 4;   // column groups per CTA (x slice of 512 values)
constexpr int kGvStride = kGvThreads;

constexpr size_t kGvLut = 65536;
constexpr size_t kGvCt = 4096;
constexpr size_t kGvWords = 16 * kGvStride * 4;
constexpr size_t kGvNib = 16 * kGvThreads * 4;

template <int B>
constexpr size_t gv_smem()
{
    return kGvLut + kGvCt + kGvWords + kGvNib + (size_t)kGvColGroups * kG * B * 4;
}

template <int B>
__global__ void __launch_bounds__(kGvThreads, 1)
    gemv_kernel(const DevTables* __restrict__ tb, const uint8_t* __restrict__ blocks, int64_t rows,
                int64_t gpr, const uint16_t* __restrict__ x, int batch, int64_t cols,
                float* __restrict__ y)
{
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t* s_lut = smem;
    float* s_Ct = reinterpret_cast<float*>(smem + kGvLut);
    uint32_t* s_w = reinterpret_cast<uint32_t*>(smem + kGvLut + kGvCt);
    uint32_t* s_nib = s_w + 16 * kGvStride;
    float* s_x = reinterpret_cast<float*>(s_nib + 16 * kGvThreads);  // [k][B]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    const int64_t g0 = (int64_t)blockIdx.y * kGvColGroups;
    const int ng = (int)min((int64_t)kGvColGroups, gpr - g0);
    {
        stage_tables<kGvThreads>(tb, s_lut, s_Ct, tid);
        for (int i = tid; i < kGvColGroups * kG * B; i += kGvThreads) {
            int k = i / B, bb = i - k * B;
            float v = 0.0f;
            if (bb < batch && k < ng * kG) v = bf16_bits_to_f32(x[(int64_t)bb * cols + g0 * kG + k]);
            s_x[i] = v;
        }
    }
    const float S_t = tb->S_t;
    __syncthreads();

    const int64_t row = ((int64_t)blockIdx.x * kGvWarps + warp) * 32 + lane;
    const bool row_ok = row < rows;
    uint32_t* ws = s_w + tid;
    uint32_t* nibs = s_nib + tid;
    float acc[B];
#pragma unroll
    for (int bb = 0; bb < B; ++bb) acc[bb] = 0.0f;

    for (int gi = 0; gi < ng; ++gi) {
        const float* xs = s_x + gi * kG * B;
        uint4 q0 = make_uint4(0, 0, 0, 0), q1 = q0, q2 = q0, q3 = q0;
        if (row_ok) {
            const uint8_t* src = blocks + (row * gpr + g0 + gi) * ECCO_BLOCK_BYTES;
            q0 = ldg_nc_v4(src);
            q1 = ldg_nc_v4(src + 16);
            q2 = ldg_nc_v4(src + 32);
            q3 = ldg_nc_v4(src + 48);
        }
        const uint32_t code = q0.x & 0xffu;
        const int p = (int)((q0.x >> 8) & 63u);
        // a row past the end or a null scale contributes zeros
        const float s = (row_ok && !scale_code_is_null(code)) ? __fmul_rn(S_t, e4m3_to_f32(code)) : 0.0f;
        stage_words(ws, kGvStride, q0, q1, q2, q3);
        const ValuePlanes vp = make_planes(s, s_Ct, p);
        const uint8_t* lut = s_lut + ((q0.x >> 8) & 255u) * 256;

        Stream st{q0.x, q0.y, kHdrBits, 2, kPayloadBits};
#pragma unroll 1
        for (int c = 0; c < 16; ++c) {
            uint32_t w[4];
            nibs[c * kGvThreads] = chunk_values(st, lut, ws, kGvStride, vp, w);
            const float* xk = xs + c * 8 * B;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float v = __uint_as_float((j & 1) ? (w[j >> 1] & 0xffff0000u) : (w[j >> 1] << 16));
#pragma unroll
                for (int bb = 0; bb < B; ++bb) acc[bb] = fmaf(v, xk[j * B + bb], acc[bb]);
            }
        }
        if (s != 0.0f && st.room >= 0) {  // outlier records replace their element's value
            const int n = min(kMaxRec, st.room / kRecBits);
            const int at0 = kBlockBits - st.room;
            for (int k = n - 1; k >= 0; --k) {  // the last record of an element wins
                uint32_t rec = read_record(ws, kGvStride, at0 + k * kRecBits);
                int i = (int)(rec & 127u);
                bool later = false;
                for (int k2 = k + 1; k2 < n; ++k2)
                    later = later || ((int)(read_record(ws, kGvStride, at0 + k2 * kRecBits) & 127u) == i);
                if (later) continue;
                float nv = bf16_bits_to_f32(f32_to_bf16_bits(__fmul_rn(s, __ldg(&tb->o_of_q[rec >> 7]))));
                uint32_t osym = (nibs[(i >> 3) * kGvThreads] >> (4 * (i & 7))) & 15u;
                uint32_t ow = (osym < 8) ? ((osym < 4) ? vp.lo[0] : vp.lo[1]) : ((osym < 12) ? vp.lo[2] : vp.lo[3]);
                uint32_t oh = (osym < 8) ? ((osym < 4) ? vp.hi[0] : vp.hi[1]) : ((osym < 12) ? vp.hi[2] : vp.hi[3]);
                uint32_t sh = 8 * (osym & 3);
                float ov = __uint_as_float((((ow >> sh) & 0xffu) | (((oh >> sh) & 0xffu) << 8)) << 16);
                float dv = nv - ov;
                const float* xi = xs + i * B;
#pragma unroll
                for (int bb = 0; bb < B; ++bb) acc[bb] = fmaf(dv, xi[bb], acc[bb]);
            }
        }
    }
    if (row_ok) {
#pragma unroll
        for (int bb = 0; bb < B; ++bb)
            if (bb < batch) atomicAdd(&y[(int64_t)bb * rows + row], acc[bb]);
    }
}

template <int B>
cudaError_t run_gemv(const ecco_tables* t, const uint8_t* blocks, int64_t rows, int64_t cols,
                     const uint16_t* x, int batch, float* y, cudaStream_t s)
{
    static int configured_dev = -1;
    if (configured_dev != t->device) {
        cudaError_t e = cudaFuncSetAttribute(gemv_kernel<B>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)gv_smem<B>());
        if (e != cudaSuccess) return e;
        configured_dev = t->device;
    }
    cudaError_t e = cudaMemsetAsync(y, 0, sizeof(float) * (size_t)batch * (size_t)rows, s);
    if (e != cudaSuccess) return e;
    const int64_t gpr = cols / kG;
    dim3 grid((unsigned)((rows + kGvThreads - 1) / kGvThreads),
              (unsigned)((gpr + kGvColGroups - 1) / kGvColGroups));
    gemv_kernel<B><<<grid, kGvThreads, gv_smem<B>(), s>>>(t->d, blocks, rows, gpr, x, batch, cols, y);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemv(const ecco_tables* t, const uint8_t* blocks, int64_t rows, int64_t cols,
                        const uint16_t* x, int batch, float* y, cudaStream_t s)
{
    if (batch == 1) return run_gemv<1>(t, blocks, rows, cols, x, batch, y, s);
    if (batch <= 4) return run_gemv<4>(t, blocks, rows, cols, x, batch, y, s);
    return launch_gemm_tc(t, blocks, rows, cols, x, batch, y, s);  // tensor cores, ecco_gemm_tc.cu
}

}  // namespace ecco
