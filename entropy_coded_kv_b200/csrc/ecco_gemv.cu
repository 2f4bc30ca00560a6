// Fused decode + matrix-vector product on CUDA cores.
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
#include "ecco_internal.cuh"

namespace ecco {
namespace {

constexpr int kGvThreads = 512;
constexpr int kGvWarps = kGvThreads / 32;
constexpr int kGvColGroups = 4;   // column groups per CTA (x slice of 512 values)
constexpr int kGvStride = kGvThreads + 2;

constexpr size_t kGvLut = 65536;
constexpr size_t kGvCt = 4096;
constexpr size_t kGvVt = 16 * kGvThreads * 4;
constexpr size_t kGvWords = 16 * kGvStride * 4;
constexpr size_t kGvNib = 16 * kGvThreads * 4;

template <int B>
constexpr size_t gv_smem()
{
    return kGvLut + kGvCt + kGvVt + kGvWords + kGvNib + (size_t)kGvColGroups * kG * B * 4;
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
    float* s_vt = reinterpret_cast<float*>(smem + kGvLut + kGvCt);
    uint32_t* s_w = reinterpret_cast<uint32_t*>(smem + kGvLut + kGvCt + kGvVt);
    uint32_t* s_nib = s_w + 16 * kGvStride;
    float* s_x = reinterpret_cast<float*>(s_nib + 16 * kGvThreads);  // [k][B]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    const int64_t g0 = (int64_t)blockIdx.y * kGvColGroups;
    const int ng = (int)min((int64_t)kGvColGroups, gpr - g0);
    {
        const uint4* a = reinterpret_cast<const uint4*>(&tb->lut[0][0]);
        uint4* b = reinterpret_cast<uint4*>(s_lut);
        for (int i = tid; i < (int)(kGvLut / 16); i += kGvThreads) b[i] = a[i];
        const uint4* c = reinterpret_cast<const uint4*>(&tb->Ct[0][0]);
        uint4* e = reinterpret_cast<uint4*>(s_Ct);
        for (int i = tid; i < (int)(kGvCt / 16); i += kGvThreads) e[i] = c[i];
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
    float* vt = s_vt + tid;
    uint32_t* ws = s_w + tid;
    uint32_t* nib = s_nib + tid;
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
        const int cb = (int)((q0.x >> 8) & 255u);
        const bool live = row_ok && !scale_code_is_null(code);
        ws[2 * kGvStride] = q0.z;
        ws[3 * kGvStride] = q0.w;
        ws[4 * kGvStride] = q1.x;
        ws[5 * kGvStride] = q1.y;
        ws[6 * kGvStride] = q1.z;
        ws[7 * kGvStride] = q1.w;
        ws[8 * kGvStride] = q2.x;
        ws[9 * kGvStride] = q2.y;
        ws[10 * kGvStride] = q2.z;
        ws[11 * kGvStride] = q2.w;
        ws[12 * kGvStride] = q3.x;
        ws[13 * kGvStride] = q3.y;
        ws[14 * kGvStride] = q3.z;
        ws[15 * kGvStride] = q3.w;
        const float s = __fmul_rn(S_t, e4m3_to_f32(code));
#pragma unroll
        for (int j = 0; j < 16; ++j)
            vt[j * kGvThreads] = live ? bf16_bits_to_f32(f32_to_bf16_bits(__fmul_rn(s, s_Ct[j * kNPat + p]))) : 0.0f;

        const uint8_t* lut = s_lut + cb * 256;
        uint32_t lo = q0.x, hi = q0.y;
        int b = kHdrBits, widx = 2, room = kBlockBits - kHdrBits;
        bool valid = true;
#pragma unroll 1
        for (int c = 0; c < 16; ++c) {
            uint32_t nb = 0;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                if (b >= 32) {
                    lo = hi;
                    hi = (widx < 16) ? ws[widx * kGvStride] : 0u;
                    widx++;
                    b -= 32;
                }
                uint32_t cur = __funnelshift_r(lo, hi, b);
                int used = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t e = lut[cur & 0xffu];
                    int len = (int)(e >> 4);
                    cur >>= len;
                    used += len;
                    valid = valid && (used <= room);
                    uint32_t sym = e & 15u;
                    nb |= sym << (4 * (half * 4 + j));
                    float v = valid ? vt[sym * kGvThreads] : 0.0f;
                    const float* xk = xs + (c * 8 + half * 4 + j) * B;
#pragma unroll
                    for (int bb = 0; bb < B; ++bb) acc[bb] = fmaf(v, xk[bb], acc[bb]);
                }
                b += used;
                room -= used;
            }
            nib[c * kGvThreads] = nb;
        }
        if (live && valid) {
            int L = kPayloadBits - room;
            int n = min(kMaxRec, room / kRecBits);
            int at0 = kHdrBits + L;
            for (int k = n - 1; k >= 0; --k) {  // last record of an element wins
                int at = at0 + k * kRecBits;
                int wi = at >> 5;
                uint32_t rec = __funnelshift_r(ws[wi * kGvStride], (wi + 1 < 16) ? ws[(wi + 1) * kGvStride] : 0u,
                                               at & 31) & 0x7fffu;
                int i = (int)(rec & 127u);
                bool later = false;
                for (int k2 = k + 1; k2 < n; ++k2) {
                    int a2 = at0 + k2 * kRecBits;
                    int w2 = a2 >> 5;
                    uint32_t r2 = __funnelshift_r(ws[w2 * kGvStride], (w2 + 1 < 16) ? ws[(w2 + 1) * kGvStride] : 0u,
                                                  a2 & 31);
                    later = later || ((int)(r2 & 127u) == i);
                }
                if (later) continue;
                int qv = (int)(int8_t)(uint8_t)(rec >> 7);
                float nv = bf16_bits_to_f32(f32_to_bf16_bits(__fmul_rn(s, __fdiv_rn((float)qv, 127.0f))));
                uint32_t osym = (nib[(i >> 3) * kGvThreads] >> (4 * (i & 7))) & 15u;
                float ov = vt[osym * kGvThreads];
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
    return run_gemv<16>(t, blocks, rows, cols, x, batch, y, s);
}

}  // namespace ecco
