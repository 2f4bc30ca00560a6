// Fused decode + matrix-vector product on CUDA cores (batch 1..4; larger
// batches go to the tensor-core kernel in ecco_gemm_tc.cu).
//
// y[b][r] = sum_k W~[r][k] * x[b][k], W~ the decoded matrix, never written to
// memory (the review page's figure list: "Normalized Memory Requests for a
// GEMM Kernel" -- compressed weights are what crosses the memory bus).
//
// Layout of the work: an item is one strip of 32 rows (a warp, a lane per
// row) x one column group, numbered column group by column group.  Each CTA
// (one per SM, resident) owns a balanced, contiguous range of items, so CTAs
// differ by at most one item (whole units of one row per thread would leave
// the SMs that own one unit fewer idle for a quarter of the launch at the
// 14336 x 4096 shape).  When the range lies in one x window its warps claim
// items from a shared counter as they finish; otherwise they run it in rounds
// of one item per warp.  All lanes of a warp need the same x[k] at every step
// (a broadcast shared-memory read); x is staged in windows of 32 column
// groups, restaged when a round reaches past the window.  Each lane decodes
// its row's block serially (one lookup per symbol, as in the decoder) and
// multiplies every decoded bf16 value, exactly, in fp32 against the batch of
// x.  An outlier record replaces the value of its element, so its
// contribution is corrected by (new - old) * x, with the old symbol kept in
// shared memory.  Each item's row sums are added to y with fp32 atomics.
#include "ecco_block.cuh"

namespace ecco {
namespace {

constexpr int kGvWin = 32;        // column groups of x staged at a time (4096 values)
constexpr size_t kGvLut = 65536;
constexpr size_t kGvCt = 4096;

// Threads per CTA (= rows per unit): batch 1 fits the decoder's 1024 threads
// (64 registers); larger batches need more registers for the accumulators.
template <int B>
constexpr int gv_threads()
{
    return B == 1 ? 1024 : 512;
}

template <int B>
constexpr size_t gv_smem()
{
    return kSmemAlign + kGvLut + kGvCt + (size_t)16 * gv_threads<B>() * 4 * 2 + (size_t)kGvWin * kG * B * 4;
}

template <int B>
__global__ void __launch_bounds__(gv_threads<B>(), 1)
    gemv_kernel(const DevTables* __restrict__ tb, const uint8_t* __restrict__ blocks, int64_t rows,
                int64_t gpr, const uint16_t* __restrict__ x, int batch, int64_t cols,
                float* __restrict__ y)
{
    constexpr int kGvThreads = gv_threads<B>(), kGvStride = kGvThreads;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t* smem = aligned_smem(smem_raw);
    uint8_t* s_lut = smem;
    float* s_Ct = reinterpret_cast<float*>(smem + kGvLut);
    uint32_t* s_w = reinterpret_cast<uint32_t*>(smem + kGvLut + kGvCt);
    uint32_t* s_nib = s_w + 16 * kGvStride;
    float* s_x = reinterpret_cast<float*>(s_nib + 16 * kGvThreads);  // [k][B], one window
    const int tid = threadIdx.x;

    stage_tables<kGvThreads>(tb, s_lut, s_Ct, tid);
    const float S_t = tb->S_t;
    constexpr int kWarps = kGvThreads / 32;
    const int lane = tid & 31, warp = tid >> 5;
    const int64_t strips = (rows + 31) / 32;
    const int64_t items = strips * gpr;  // item q: column group q / strips, strip q % strips
    const int64_t qa = items * blockIdx.x / gridDim.x, qb = items * (blockIdx.x + 1) / gridDim.x;

    uint32_t* ws = s_w + tid;
    uint32_t* nibs = s_nib + tid;
    int64_t win0 = -1;  // first column group of the staged x window

    // One item: this warp's 32 rows of column group q / strips, x from the
    // staged window.
    auto do_item = [&](int64_t q) {
        const int64_t gcol = q / strips;
        const int64_t row = (q - gcol * strips) * 32 + lane;
        const bool row_ok = row < rows;
        const float* xs = s_x + (gcol - win0) * kG * B;
        float acc[B];
#pragma unroll
        for (int bb = 0; bb < B; ++bb) acc[bb] = 0.0f;
        {
        uint4 q0 = make_uint4(0, 0, 0, 0), q1 = q0, q2 = q0, q3 = q0;
        if (row_ok) {
            const uint8_t* src = blocks + (row * gpr + gcol) * ECCO_BLOCK_BYTES;
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
        const uint32_t lkey = lut_key(s_lut, (q0.x >> 8) & 255u);

        Stream st{q0.x, q0.y, kHdrBits, 2, kPayloadBits};
#pragma unroll 1
        for (int c = 0; c < 16; ++c) {
            uint32_t w[4];
            nibs[c * kGvThreads] = chunk_values(st, lkey, ws, kGvStride, vp, w);
            // the chunk's 8 x B inputs as 16-byte broadcast loads (one L1 wavefront each)
            float xk[8 * B];
#pragma unroll
            for (int v4 = 0; v4 < 2 * B; ++v4) {
                const float4 t = reinterpret_cast<const float4*>(xs + c * 8 * B)[v4];
                xk[4 * v4] = t.x;
                xk[4 * v4 + 1] = t.y;
                xk[4 * v4 + 2] = t.z;
                xk[4 * v4 + 3] = t.w;
            }
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
            // Newest first: the last record of an element wins, so an element
            // already seen (128-bit mask) is skipped.
            uint32_t seen0 = 0u, seen1 = 0u, seen2 = 0u, seen3 = 0u;
            for (int k = n - 1; k >= 0; --k) {
                uint32_t rec = read_record(ws, kGvStride, at0 + k * kRecBits);
                int i = (int)(rec & 127u);
                const uint32_t bit = 1u << (i & 31), q = (uint32_t)i >> 5;
                const uint32_t was = (q == 0u ? seen0 : q == 1u ? seen1 : q == 2u ? seen2 : seen3) & bit;
                seen0 |= (q == 0u) ? bit : 0u;
                seen1 |= (q == 1u) ? bit : 0u;
                seen2 |= (q == 2u) ? bit : 0u;
                seen3 |= (q == 3u) ? bit : 0u;
                if (was) continue;
                float nv = bf16_bits_to_f32(f32_to_bf16_bits(__fmul_rn(s, q_over_127((int)(int8_t)(uint8_t)(rec >> 7)))));
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
    };

    __shared__ unsigned int s_next;  // items of the CTA's range claimed so far
    if (qb > qa && (qb - 1) / strips - qa / strips < kGvWin) {
        // The whole range lies in one x window: staged once, and the warps
        // claim items one at a time as they finish, so the range's last items
        // go to the warps that are free first, not to fixed warps in a short
        // last round.
        const int64_t k0 = (qa / strips) * kG;
        const int nk = (int)min((int64_t)kGvWin * kG, cols - k0);
        for (int i = tid; i < kGvWin * kG * B; i += kGvThreads) {
            const int k = i / B, bb = i - k * B;
            s_x[i] = (bb < batch && k < nk) ? bf16_bits_to_f32(x[(int64_t)bb * cols + k0 + k]) : 0.0f;
        }
        win0 = qa / strips;
        if (tid == 0) s_next = 0u;
        __syncthreads();  // window, tables and counter ready
        for (;;) {
            unsigned int c = 0;
            if (lane == 0) c = atomicAdd(&s_next, 1u);
            c = __shfl_sync(0xffffffffu, c, 0);
            if (qa + (int64_t)c >= qb) break;
            do_item(qa + (int64_t)c);
        }
        return;
    }

    for (int64_t q0 = qa; q0 < qb; q0 += kWarps) {
        // the round's column groups must lie in the window (uniform across the CTA)
        const int64_t g_first = q0 / strips, g_last = (min(q0 + kWarps, qb) - 1) / strips;
        if (win0 < 0 || g_first < win0 || g_last >= win0 + kGvWin) {
            __syncthreads();  // the previous window is no longer read (and the tables are staged)
            win0 = g_first;
            const int64_t k0 = win0 * kG;
            const int nk = (int)min((int64_t)kGvWin * kG, cols - k0);
            for (int i = tid; i < kGvWin * kG * B; i += kGvThreads) {
                const int k = i / B, bb = i - k * B;
                s_x[i] = (bb < batch && k < nk) ? bf16_bits_to_f32(x[(int64_t)bb * cols + k0 + k]) : 0.0f;
            }
            __syncthreads();
        }
        const int64_t q = q0 + warp;
        if (q >= qb) continue;  // this warp has no item in the CTA's short last round
        do_item(q);
    }
}

template <int B>
cudaError_t run_gemv(const ecco_tables* t, const uint8_t* blocks, int64_t rows, int64_t cols,
                     const uint16_t* x, int batch, float* y, cudaStream_t s)
{
    static std::atomic<uint64_t> configured{0};
    if (cudaError_t e0 = set_max_smem_once(configured, (const void*)gemv_kernel<B>, gv_smem<B>()); e0 != cudaSuccess)
        return e0;
    cudaError_t e = cudaMemsetAsync(y, 0, sizeof(float) * (size_t)batch * (size_t)rows, s);
    if (e != cudaSuccess) return e;
    const int64_t gpr = cols / kG;
    const int64_t items = (rows + 31) / 32 * gpr;  // 32-row strips x column groups
    const int64_t per_cta = gv_threads<B>() / 32;   // one item per warp per round
    const int64_t want = (items + per_cta - 1) / per_cta;
    const int grid = (int)(want < device_sm_count() ? want : device_sm_count());  // one resident CTA per SM
    gemv_kernel<B><<<grid, gv_threads<B>(), gv_smem<B>(), s>>>(t->d, blocks, rows, gpr, x, batch, cols, y);
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
