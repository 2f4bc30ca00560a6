// Fused decode + batched matrix-vector product on the 5th-generation tensor
// cores (tcgen05), for batch 5..16.
//
// y[b][r] = sum_k W~[r][k] x[b][k]: with a batch of activations the product
// is a real dense contraction (M = rows, N = batch, K = cols), so the decoded
// weights go to the tensor cores instead of 16 FMAs per weight on CUDA cores.
// (Review page, figure list: "Normalized Memory Requests for a GEMM Kernel" --
// only compressed weights cross the memory bus.)
//
// Work units are (row tile of 768 rows, one column group of 128 values); each
// CTA (768 threads, one per SM) owns a balanced, contiguous range of units in
// row-tile-major order, so consecutive units share a row tile and its
// accumulators.  When the units do not divide evenly over the CTAs and the
// remainder is small, the remainder is not handed out whole (one more round
// on a few SMs, the rest idle): its units are cut into warp steps of 32 rows,
// spread over the CTAs, and in each CTA the warps that finish their whole
// units first claim them.  Thread t decodes row t's block of the unit with the block
// walker of ecco_block.cuh.  The walk's speed comes from the warps running
// freely (its latency is hidden by the other warps), so every warp feeds the
// tensor cores on its own, with no barrier between warps inside a unit:
//   - the 4 warps w = 4j..4j+3 share A tile buffers j (double buffered), 128
//     rows x 16 values (one K = 16 slice, K-major, no swizzle: 8-row x
//     16-byte core matrices); warp w writes rows 32 (w & 3) .. + 31;
//   - lane 0 of warp w then issues tcgen05.mma (M = 128, N = 16, K = 16, bf16
//     in, fp32 accumulate) on the whole tile into warp w's own 16 columns of
//     tensor memory, and commits it to the warp's mbarrier for that buffer;
//   - row r of the product depends on row r of A only, so the rows the other
//     three warps are writing (or have overwritten) reach only lanes of warp
//     w's columns that warp w never reads: it reads back lanes 32 (w & 3) ..
//     + 31, the lanes its own rows produced;
//   - a warp writes a buffer again only after its own MMA that read it has
//     completed.
// x of a unit's column group is its B operand, in a ring of 4 slots that all
// threads fill two units ahead: a slot's "full" mbarrier completes when every
// thread has written its share (and it is waited on before the unit's first
// MMA); its "free" mbarrier completes when every warp's MMAs of the unit that
// used it have finished and every warp has read its record corrections from
// it (each warp's lane 0 commits to it after its last MMA of the unit, and
// arrives on it after the records), and it is waited on before the slot is
// refilled.  So no
// barrier holds the warps together inside or between units: a warp can run up
// to two units ahead of the slowest.  The centroids are read through the
// read-only cache; shared memory holds the decode tables, the stream words,
// the decoded symbols (for the records), A and the x ring.
//
// Outlier records are known only at the end of a block's stream, after its
// slices went to the tensor cores, so their effect is added on CUDA cores as
// (new - old) * x.  When a CTA's units move to the next row tile (and at the
// end) each row's accumulators plus corrections are added to y with fp32
// atomics (a row tile is split over a few CTAs).
//
// Every wait on an mbarrier is bounded.  A wait that gives up counts itself
// (ecco_device_timeouts) and raises a host-visible flag; its warp then issues
// no more MMAs and writes nothing more to y (the launch's y is incomplete and
// the next tensor-core ecco_decode_gemv call returns ECCO_ERR_TIMEOUT); at the
// end the CTA waits once more (bounded) for the MMAs it committed, frees its
// tensor memory and returns.
#include <mutex>

#include "ecco_block.cuh"

namespace ecco {

__device__ unsigned int g_timeouts = 0;

namespace {

constexpr int kTcThreads = 768;
constexpr int kTcTiles = kTcThreads / 128;   // M-tiles of 128 rows
constexpr int kTcStride = kTcThreads;        // word k of thread t's arrays at k * stride + t
constexpr int kSliceBytes = 128 * 16 * 2;    // one 128 x 16 bf16 A slice
constexpr int kBSliceBytes = 16 * 16 * 2;    // one 16 x 16 bf16 B slice
constexpr int kBBytes = 8 * kBSliceBytes;    // x of one column group: 8 slices
constexpr uint32_t kSpinLimit = 1u << 22;    // polls; with the back-off below, well under a second

constexpr size_t kOffLut = 0;
constexpr size_t kOffWords = kOffLut + 65536;
constexpr size_t kOffNib = kOffWords + (size_t)16 * kTcStride * 4;
constexpr size_t kOffA = kOffNib + (size_t)16 * kTcThreads * 4;
constexpr size_t kOffB = kOffA + (size_t)kTcTiles * 2 * kSliceBytes;
constexpr int kBSlots = 4;                   // x ring: filled two units ahead
constexpr size_t kOffBar = kOffB + (size_t)kBSlots * kBBytes;
constexpr int kTcWarps = kTcThreads / 32;
// [warp][2]: the warp's MMAs on A buffer 0 / 1; then x ring full[4], free[4]
constexpr int kNumBars = 2 * kTcWarps + 2 * kBSlots;
constexpr size_t kTcSmem = kOffBar + (size_t)kNumBars * 8 + 16 + kSmemAlign;
constexpr uint32_t kTmemCols = 512;     // 24 warps x 16 fp32 columns, rounded up to a power of 2

// Instruction descriptor: D fp32 (bits 4-5 = 1), A and B bf16 (bits 7-9, 10-12
// = 1), both K-major, N >> 3 in bits 17-22, M >> 4 in bits 24-28.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((16u >> 3) << 17) | ((128u >> 4) << 24);

// Shared-memory matrix descriptor, K-major without swizzle: start >> 4,
// leading byte offset (between the two 8-element K halves) 128 B, stride byte
// offset (between 8-row groups) 256 B, descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr)
{
    return (uint64_t)((addr >> 4) & 0x3fffu) | ((uint64_t)(128u >> 4) << 16) | ((uint64_t)(256u >> 4) << 32) |
           (1ull << 46);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

// Waits for the phase with the given parity to complete: non-blocking polls,
// with a short sleep after the first few, at most kSpinLimit of them.
// Returns false if it gave up, after counting the timeout and raising `flag`
// (host-visible) when there is one.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* flag)
{
    const uint32_t a = smem_u32(bar);
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
        if (i >= 16) __nanosleep(64);
    }
    atomicAdd(&g_timeouts, 1u);
    if (flag) {
        *reinterpret_cast<volatile int*>(flag) = 1;
        __threadfence_system();
    }
    return false;
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Byte offset of element (row, k) inside a 128 x 16 K-major slice.
__device__ __forceinline__ uint32_t a_offset(int row, int khalf)
{
    return (uint32_t)((row >> 3) * 256 + khalf * 128 + (row & 7) * 16);
}

// Byte offset of x[b][k] (k within a 16-wide slice) inside a 16 x 16 B slice.
__device__ __forceinline__ uint32_t b_offset(int b, int kk)
{
    return (uint32_t)((b >> 3) * 256 + (kk >> 3) * 128 + (b & 7) * 16 + (kk & 7) * 2);
}

struct TcArgs {
    const DevTables* tb;
    const uint8_t* blocks;
    const uint16_t* x;
    float* y;
    int* flag;  // host-visible timeout flag (mapped pinned memory), or null
    int64_t rows, gpr, cols, units;  // units: whole units handed out to the CTAs
    int64_t tail_steps;              // warp steps of the units left over (0: none)
    int batch;
    bool wide;  // blocks 32-byte aligned
};

__global__ void __launch_bounds__(kTcThreads, 1) gemm_tc_kernel(const __grid_constant__ TcArgs A)
{
    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint8_t* smem = aligned_smem(smem_raw);
    uint8_t* s_lut = smem + kOffLut;
    uint32_t* s_w = reinterpret_cast<uint32_t*>(smem + kOffWords);
    uint32_t* s_nib = reinterpret_cast<uint32_t*>(smem + kOffNib);
    uint8_t* s_A = smem + kOffA;
    uint8_t* s_B = smem + kOffB;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kOffBar + kNumBars * 8);
    unsigned int* s_next = reinterpret_cast<unsigned int*>(s_tmem + 1);  // leftover steps claimed so far

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tile = warp >> 2;               // 4 warps per 128-row tile
    const int trow = (warp & 3) * 32 + lane;  // row inside the tile = TMEM lane
    const DevTables* tb = A.tb;
    const float* Ct = &tb->Ct[0][0];

    const int64_t u0 = A.units * blockIdx.x / gridDim.x, u1 = A.units * (blockIdx.x + 1) / gridDim.x;

    stage_lut<kTcThreads>(tb, s_lut, tid);
    uint64_t* bar_full = &bars[2 * kTcWarps];
    uint64_t* bar_free = &bars[2 * kTcWarps + kBSlots];
    if (tid == 0) {
        *s_next = 0u;
        for (int i = 0; i < 2 * kTcWarps; ++i) mbar_init(&bars[i], 1);
        for (int i = 0; i < kBSlots; ++i) {
            mbar_init(&bar_full[i], kTcThreads);  // every thread writes a share of x
            // every warp twice: its lane 0 commits (the MMAs that read the slot are
            // done) and arrives (its lanes have read their record corrections)
            mbar_init(&bar_free[i], 2 * kTcWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_tmem)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem_d = *s_tmem + (uint32_t)(16 * warp);  // this warp's 16 fp32 columns
    const uint32_t taddr = tmem_d + ((uint32_t)((warp & 3) * 32) << 16);  // ... at its own lanes
    const float S_t = tb->S_t;

    uint32_t* ws = s_w + tid;
    uint32_t* nibs = s_nib + tid;
    uint8_t* A0 = s_A + tile * 2 * kSliceBytes;
    const bool issuer = lane == 0;
    uint64_t* bar_buf = &bars[warp * 2];
    float corr[16];
#pragma unroll
    for (int b = 0; b < 16; ++b) corr[b] = 0.0f;
    bool ok = true;      // uniform in the warp after every slice
    int t = 0;           // slices so far (the A buffer is t & 1)
    bool acc = false;    // the warp's accumulators hold a partial sum
    const int64_t nu = u1 - u0;
    int64_t tile_row = (nu > 0) ? u0 / A.gpr : 0;
    // Leftover units (when the units do not divide over the CTAs) are split
    // into warp steps of 32 rows, kTcWarps per unit, and spread evenly: this
    // CTA's steps [ts0, ts1) belong to at most two leftover units, its local
    // units nu .. nl - 1 (their x goes through the ring like any unit's).
    const int64_t ts0 = A.tail_steps * blockIdx.x / gridDim.x, ts1 = A.tail_steps * (blockIdx.x + 1) / gridDim.x;
    const int64_t tl0 = ts0 / kTcWarps;
    const int64_t nl = nu + ((ts1 > ts0) ? (ts1 - 1) / kTcWarps - tl0 + 1 : 0);

    // This thread's share of x for local unit l into its ring slot (l % 4),
    // after the unit that used the slot before (l - 4) has no MMA left; then
    // it announces the share on the slot's "full" mbarrier.
    auto stage_x = [&](int64_t l) {
        const int slot = (int)(l % kBSlots);
        if (l >= kBSlots && ok) ok = mbar_wait(&bar_free[slot], (uint32_t)((l / kBSlots - 1) & 1), A.flag);
        const int64_t g = (l < nu ? u0 + l : A.units + tl0 + (l - nu)) % A.gpr;
        uint8_t* Bw = s_B + slot * kBBytes;
        for (int e = tid; e < 16 * kG; e += kTcThreads) {
            const int b = e & 15, k = e >> 4;
            const uint16_t v = (b < A.batch) ? A.x[(int64_t)b * A.cols + g * kG + k] : (uint16_t)0;
            *reinterpret_cast<uint16_t*>(Bw + (k >> 4) * kBSliceBytes + b_offset(b, k & 15)) = v;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // written by generic stores
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&bar_full[slot])) : "memory");
    };
    // Waits until this warp's MMAs issued so far have completed (the commit of
    // the last slice completes after all of them).
    auto drain = [&]() {
        if (t >= 1 && ok) ok = mbar_wait(&bar_buf[(t - 1) & 1], (uint32_t)(((t - 1) >> 1) & 1), A.flag);
    };
    // Adds each thread's row of its warp's accumulators (plus the record
    // corrections) to y and starts the next row tile from zero.  Per warp.
    auto flush = [&](int64_t rt, int rb) {
        drain();
        ok = __all_sync(0xffffffffu, ok);
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        uint32_t v[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, "
            "[%16];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
            : "r"(taddr));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        const int64_t row = rt * kTcThreads + rb + lane;
        if (ok && acc && row < A.rows) {
#pragma unroll
            for (int b = 0; b < 16; ++b)
                if (b < A.batch) atomicAdd(&A.y[(int64_t)b * A.rows + row], __uint_as_float(v[b]) + corr[b]);
        }
#pragma unroll
        for (int b = 0; b < 16; ++b) corr[b] = 0.0f;
        acc = false;
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    };

    // One unit's work for this warp: its 32 rows rt * 768 + rb .. + 31 of
    // column group g, x in ring slot l % 4.
    auto run_unit = [&](int64_t l, int64_t rt, int64_t g, int rb) {
        const int slot = (int)(l % kBSlots);
        const uint8_t* B = s_B + slot * kBBytes;

        // ---- this thread's row block (and the next unit's on its way to L2)
        const int64_t row = rt * kTcThreads + rb + lane;
        const bool row_ok = row < A.rows;
        if (l + 1 < nu) {  // the next unit: the next column group, or the next row tile's first
            const bool wrap = g + 1 == A.gpr;
            const int64_t rn = row + (wrap ? kTcThreads : 0), gn = wrap ? 0 : g + 1;
            if (rn < A.rows)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(A.blocks + (rn * A.gpr + gn) * ECCO_BLOCK_BYTES));
        }
        uint4 q0 = make_uint4(0, 0, 0, 0), q1 = q0, q2 = q0, q3 = q0;
        if (row_ok) {
            const uint8_t* src = A.blocks + (row * A.gpr + g) * ECCO_BLOCK_BYTES;
            if (A.wide) {  // 32-byte aligned blocks: two 32-byte loads
                ldg_nc_v8(src, q0, q1);
                ldg_nc_v8(src + 32, q2, q3);
            } else {
                q0 = ldg_nc_v4(src);
                q1 = ldg_nc_v4(src + 16);
                q2 = ldg_nc_v4(src + 32);
                q3 = ldg_nc_v4(src + 48);
            }
        }
        const uint32_t code = q0.x & 0xffu;
        const int p = (int)((q0.x >> 8) & 63u);
        // a row past the end or a null scale contributes zeros
        const float s = (row_ok && !scale_code_is_null(code)) ? __fmul_rn(S_t, e4m3_to_f32(code)) : 0.0f;
        stage_words(ws, kTcStride, q0, q1, q2, q3);
        const ValuePlanes vp = make_planes<true>(s, Ct, p);
        const uint32_t lkey = lut_key(s_lut, (q0.x >> 8) & 255u);
        Stream st{q0.x, q0.y, kHdrBits, 2, kPayloadBits};

#pragma unroll 1
        for (int sl = 0; sl < 8; ++sl, ++t) {
            uint32_t wa[4], wb[4];
            nibs[(2 * sl) * kTcThreads] = chunk_values(st, lkey, ws, kTcStride, vp, wa);
            nibs[(2 * sl + 1) * kTcThreads] = chunk_values(st, lkey, ws, kTcStride, vp, wb);
            const int buf = t & 1, use = t >> 1;
            if (use >= 1 && ok) ok = mbar_wait(&bar_buf[buf], (uint32_t)((use - 1) & 1), A.flag);
            if (sl == 0 && ok) ok = mbar_wait(&bar_full[slot], (uint32_t)((l / kBSlots) & 1), A.flag);
            uint8_t* Ab = A0 + buf * kSliceBytes;
            *reinterpret_cast<uint4*>(Ab + a_offset(trow, 0)) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
            *reinterpret_cast<uint4*>(Ab + a_offset(trow, 1)) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            // the warp's 32 rows are written (memory ordering among its lanes) and
            // its lanes agree that no wait gave up
            __syncwarp();
            ok = __all_sync(0xffffffffu, ok);
            if (issuer && ok) {
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint64_t ad = smem_desc(smem_u32(Ab));
                const uint64_t bd = smem_desc(smem_u32(B + sl * kBSliceBytes));
                mma_bf16(tmem_d, ad, bd, acc ? 1u : 0u);
                mma_commit(&bar_buf[buf]);
                if (sl == 7) mma_commit(&bar_free[slot]);  // the x slot is free once these MMAs are done
            }
            acc = true;
        }

        if (s != 0.0f && st.room >= 0) {  // outlier records: add (new - old) * x
            const int n = min(kMaxRec, st.room / kRecBits);
            const int at0 = kBlockBits - st.room;
            // Newest first: the last record of an element wins, so an element
            // already seen (128-bit mask) is skipped.
            uint32_t seen0 = 0u, seen1 = 0u, seen2 = 0u, seen3 = 0u;
            for (int k = n - 1; k >= 0; --k) {
                const uint32_t rec = read_record(ws, kTcStride, at0 + k * kRecBits);
                const int i = (int)(rec & 127u);
                const uint32_t bit = 1u << (i & 31), q = (uint32_t)i >> 5;
                const uint32_t was = (q == 0u ? seen0 : q == 1u ? seen1 : q == 2u ? seen2 : seen3) & bit;
                seen0 |= (q == 0u) ? bit : 0u;
                seen1 |= (q == 1u) ? bit : 0u;
                seen2 |= (q == 2u) ? bit : 0u;
                seen3 |= (q == 3u) ? bit : 0u;
                if (was) continue;
                const float nv =
                    bf16_bits_to_f32(f32_to_bf16_bits(__fmul_rn(s, q_over_127((int)(int8_t)(uint8_t)(rec >> 7)))));
                const uint32_t osym = (nibs[(i >> 3) * kTcThreads] >> (4 * (i & 7))) & 15u;
                const uint32_t ow =
                    (osym < 8) ? ((osym < 4) ? vp.lo[0] : vp.lo[1]) : ((osym < 12) ? vp.lo[2] : vp.lo[3]);
                const uint32_t oh =
                    (osym < 8) ? ((osym < 4) ? vp.hi[0] : vp.hi[1]) : ((osym < 12) ? vp.hi[2] : vp.hi[3]);
                const uint32_t sh = 8 * (osym & 3);
                const float ov = __uint_as_float((((ow >> sh) & 0xffu) | (((oh >> sh) & 0xffu) << 8)) << 16);
                const float dv = nv - ov;
                const uint8_t* Bs = B + (i >> 4) * kBSliceBytes;
#pragma unroll
                for (int b = 0; b < 16; ++b) {
                    const float xv = bf16_bits_to_f32(*reinterpret_cast<const uint16_t*>(Bs + b_offset(b, i & 15)));
                    corr[b] = fmaf(dv, xv, corr[b]);
                }
            }
        }
        __syncwarp();  // the warp's lanes are done with this unit's x slot
        if (issuer)
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&bar_free[slot])) : "memory");
    };

    for (int64_t l = 0; l < 2 && l < nl; ++l) stage_x(l);

    for (int64_t l = 0; l < nu; ++l) {
        const int64_t u = u0 + l;
        const int64_t rt = u / A.gpr, g = u - rt * A.gpr;
        if (rt != tile_row) {
            flush(tile_row, warp * 32);
            tile_row = rt;
        }
        if (l + 2 < nl) stage_x(l + 2);  // two units ahead
        run_unit(l, rt, g, warp * 32);
    }
    flush(tile_row, warp * 32);

    // The CTA's leftover steps (32 rows of a leftover unit each), claimed one
    // at a time by the warps that finish their units first, while the others
    // are still on their last.
    for (;;) {
        unsigned int c = 0;
        if (lane == 0) c = atomicAdd(s_next, 1u);
        c = __shfl_sync(0xffffffffu, c, 0);
        if ((int64_t)c >= ts1 - ts0) break;
        const int64_t j = ts0 + (int64_t)c, tu = j / kTcWarps;
        const int64_t u = A.units + tu, rt = u / A.gpr, g = u - rt * A.gpr;
        const int rb = (int)(j - tu * kTcWarps) * 32;
        run_unit(nu + (tu - tl0), rt, g, rb);
        flush(rt, rb);
    }

    // before the tensor memory is freed: the MMAs this warp committed are
    // done (bounded once more if a wait already gave up)
    if (t >= 1) mbar_wait(&bar_buf[(t - 1) & 1], (uint32_t)(((t - 1) >> 1) & 1), nullptr);
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(*s_tmem), "r"(kTmemCols)
                     : "memory");
}

// Waits on an mbarrier that nothing arrives at, with the pipeline's bounded
// wait: it gives up, counts the timeout and raises the flag.
__global__ void wait_timeout_selftest_kernel(int* flag)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        mbar_wait(&bar, 0u, flag);
    }
}

std::once_flag g_flag_once;
int* g_flag = nullptr;  // mapped pinned int shared by all devices; null if it could not be allocated

}  // namespace

int* timeout_flag()
{
    std::call_once(g_flag_once, [] {
        void* p = nullptr;
        if (cudaHostAlloc(&p, sizeof(int), cudaHostAllocMapped | cudaHostAllocPortable) == cudaSuccess) {
            *static_cast<volatile int*>(p) = 0;
            g_flag = static_cast<int*>(p);
        }
    });
    return g_flag;
}

bool timeout_raised()
{
    int* f = timeout_flag();
    return f && *reinterpret_cast<volatile int*>(f) != 0;
}

cudaError_t launch_gemm_tc(const ecco_tables* t, const uint8_t* blocks, int64_t rows, int64_t cols,
                           const uint16_t* x, int batch, float* y, cudaStream_t s)
{
    static std::atomic<uint64_t> configured{0};
    if (cudaError_t e0 = set_max_smem_once(configured, (const void*)gemm_tc_kernel, kTcSmem); e0 != cudaSuccess)
        return e0;
    cudaError_t e = cudaMemsetAsync(y, 0, sizeof(float) * (size_t)batch * (size_t)rows, s);
    if (e != cudaSuccess) return e;
    TcArgs A;
    A.tb = t->d;
    A.blocks = blocks;
    A.x = x;
    A.y = y;
    A.flag = timeout_flag();
    A.rows = rows;
    A.gpr = cols / kG;
    A.cols = cols;
    const int64_t units = (rows + kTcThreads - 1) / kTcThreads * A.gpr;
    A.batch = batch;
    A.wide = (reinterpret_cast<uintptr_t>(blocks) & 31u) == 0;
    const int64_t sms = device_sm_count();
    const int grid = (int)(units < sms ? units : sms);  // one resident CTA per SM, balanced unit ranges
    // Units left over after whole rounds would take one more round on as many
    // SMs while the rest idle; when they are at most a third of the grid they
    // are split into warp steps spread over every CTA instead.
    const int64_t left = units % grid;
    const bool split = units > grid && left * 3 <= grid;
    A.units = split ? units - left : units;
    A.tail_steps = split ? left * kTcWarps : 0;
    gemm_tc_kernel<<<grid, kTcThreads, kTcSmem, s>>>(A);
    return cudaGetLastError();
}

cudaError_t launch_wait_timeout_selftest(cudaStream_t s)
{
    wait_timeout_selftest_kernel<<<1, 32, 0, s>>>(timeout_flag());
    return cudaGetLastError();
}

}  // namespace ecco

extern "C" int ecco_device_timeouts(unsigned int* out)
{
    if (!out) return ECCO_ERR_ARG;
    if (cudaMemcpyFromSymbol(out, ecco::g_timeouts, sizeof(unsigned int)) != cudaSuccess) return ECCO_ERR_CUDA;
    if (int* f = ecco::timeout_flag()) *reinterpret_cast<volatile int*>(f) = 0;
    return ECCO_OK;
}
