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
// (flash-decoding).  One CTA of 512 threads owns a split; thread t decodes
// token split * 512 + t, one Huffman walk per block (the serial part).  The
// two contractions run on the tensor cores as warp-level mma.sync tiles (bf16
// inputs, fp32 accumulation), fed from a per-warp staging tile that holds the
// warp's 32 tokens x 32 dimensions at a time:
//   K pass  S[head][token] += Q[head][dims] . K[token][dims]^T
//           (m16n8k16: rows = query heads of the group, n = 8 tokens,
//           k = 16 dimensions; B fragments by ldmatrix from the token rows);
//   softmax CTA-wide max and sum per head; the score fragments stay in
//           registers and become the A fragments of the next product;
//   V pass  O[head][dims] += P[head][tokens] . V[tokens][dims]
//           (n = 8 dimensions, k = 16 tokens; B fragments by ldmatrix.trans).
//           P is split into bf16 hi + lo parts carried in rows 0-7 and 8-15
//           of the A operand, so O = rows 0-7 + rows 8-15 keeps p to about
//           2^-17 relative while V enters exactly.
// Outlier records change single elements after the walk: their effect is
// added as (new - old) * q on the score and p * (new - old) on the output.
// Partial (max, sum, p.V) of every split go to a caller-owned workspace; a
// second kernel merges the splits with the usual log-sum-exp rescaling.
// The staged variant reads rows the block decoder has already written and
// takes 256-token splits (8 warps per CTA) instead.
#include <atomic>

#include "ecco_block.cuh"

namespace ecco {
namespace {

constexpr int kAtThreads = 512;
constexpr int kAtWarps = kAtThreads / 32;
constexpr int kAtStride = kAtThreads;
// The staged split kernel: 8 warps, 256 tokens per split, so that three CTAs
// (row tiles and q: 71 KB of shared memory each) are resident per SM.
constexpr int kStWarps = 8;
constexpr int kStTokens = kStWarps * 32;
constexpr int kStageRow = 20;  // words per staged token row: 32 bf16 + 16 B pad (ldmatrix conflict-free)
constexpr int kHeads = 8;      // rows 0-7 of an m16 tile: the query heads of one KV head
constexpr int kQbRow = 136;    // bf16 per staged q row (padded: conflict-free fragment loads)

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
    // Staged path only: the current chunk's decoded K and V rows (bf16,
    // [B*H][cstride][128]), its first token c0 (a multiple of kStTokens) and
    // the index of its first split.
    const uint16_t* kx;
    const uint16_t* vx;
    int64_t c0, cstride;
    int split0;
};

// shared memory map (bytes)
constexpr size_t kOffLut = 0;
constexpr size_t kOffCt = kOffLut + 65536;
constexpr size_t kOffWords = kOffCt + 4096;
constexpr size_t kOffNib = kOffWords + (size_t)16 * kAtStride * 4;      // [chunk][thread] symbol nibbles
constexpr size_t kOffStage = kOffNib + (size_t)16 * kAtStride * 4;
constexpr size_t kOffX = kOffStage + (size_t)kAtWarps * 32 * kStageRow * 4;  // [warp][token][head] f32
constexpr size_t kOffQf = kOffX + (size_t)kAtWarps * 32 * kHeads * 4;         // [head][128] f32
constexpr size_t kOffQb = kOffQf + (size_t)kHeads * 128 * 4;                  // [head][kQbRow] bf16
constexpr size_t kOffRed = kOffQb + (size_t)kHeads * kQbRow * 2;              // [2][warp][head] f32
constexpr size_t kOffAcc = kOffRed + (size_t)2 * kAtWarps * kHeads * 4;       // [head][128] f32
constexpr size_t kAttnSmem = kOffAcc + (size_t)kHeads * 128 * 4 + kSmemAlign;
static_assert(kOffQb % 16 == 0 && kOffRed % 16 == 0 && kOffAcc % 16 == 0, "alignment");
// Staged path: no tables, stream words, nibbles or f32 copies of q; each
// warp's tile holds its 32 tokens' whole decoded rows (filled by cp.async),
// 272 B apart so that ldmatrix rows fall on distinct banks.  Once a warp has
// read a quarter of its V rows (dims 32 qd ..), it writes its P . V for those
// dims into the same columns of its own tile (head g in rows 2g and 2g + 1),
// and the warps' slices are summed once into the partial result (no
// shared-memory atomics: 16 warps adding into one accumulator was measured
// 9-16% slower per call).  71 KB per CTA: three CTAs of 8 warps per SM.
constexpr int kFullRow = 68;  // words per staged full row: 128 bf16 + 16 B pad
constexpr size_t kSOffTile = 0;
constexpr size_t kSOffQb = kSOffTile + (size_t)kStWarps * 32 * kFullRow * 4;
constexpr size_t kSOffRed = kSOffQb + (size_t)kHeads * kQbRow * 2;
constexpr size_t kAttnSmemStaged = kSOffRed + (size_t)2 * kStWarps * kHeads * 4 + kSmemAlign;
static_assert(kSOffQb % 16 == 0 && kSOffRed % 16 == 0, "alignment");
static_assert(3 * (kAttnSmemStaged + 1024) <= 233472, "three staged CTAs per SM");

// Tokens per chunk of the staged path: the decoded K and V rows of a chunk
// (2 x rows x chunk x 256 B) stay within kStagedScratchBytes; a multiple of
// 512 (whole splits of either kernel).  Measured on B200 ([8, 8, 4096] and [1, 8, 131072]
// caches): chunks that fit in L2 (32 MiB) are slower than one large chunk,
// because a decoder launch needs several blocks per thread to hide its serial
// walk, so the bound is set by memory use, not by L2.
constexpr int64_t kStagedScratchBytes = 1024ll << 20;

__device__ __forceinline__ void mma_bf16(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t r[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t r[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
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

// Calls f(i, new_value - old_value) once per element that an outlier record of
// an unclipped block replaces, with the element's last record (which wins).
template <class F>
__device__ __forceinline__ void for_records(const Stream& st, const uint32_t* ws, const uint32_t* nb, float s,
                                            const ValuePlanes& vp, const float* o_of_q, F f)
{
    if (s == 0.0f || st.room < kRecBits) return;
    const int n = min(kMaxRec, st.room / kRecBits);
    const int at0 = kBlockBits - st.room;
    uint32_t seen0 = 0, seen1 = 0, seen2 = 0, seen3 = 0;  // elements already given by a later record
    for (int k = n - 1; k >= 0; --k) {
        const uint32_t rec = read_record(ws, kAtStride, at0 + k * kRecBits);
        const int i = (int)(rec & 127u);
        const uint32_t bit = 1u << (i & 31);
        const uint32_t sw = (i < 64) ? ((i < 32) ? seen0 : seen1) : ((i < 96) ? seen2 : seen3);
        if (sw & bit) continue;
        if (i < 32) seen0 |= bit;
        else if (i < 64) seen1 |= bit;
        else if (i < 96) seen2 |= bit;
        else seen3 |= bit;
        const float nv = bf16_bits_to_f32(f32_to_bf16_bits(__fmul_rn(s, __ldg(o_of_q + (rec >> 7)))));
        const float ov = value_of(vp, (nb[(i >> 3) * kAtStride] >> (4 * (i & 7))) & 15u);
        f(i, nv - ov);
    }
}

// Decodes the 32 symbols of quarter `qd` of this thread's block into its row
// of the warp's staging tile; the symbols (nibbles) go to the thread's column
// nb[k * kAtStride], k = chunk, for the record pass.
__device__ __forceinline__ void decode_quarter(Stream& st, uint32_t lkey, const uint32_t* ws,
                                               const ValuePlanes& vp, uint32_t* row, uint32_t* nb, int qd)
{
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t w[4];
        nb[(qd * 4 + c4) * kAtStride] = chunk_values(st, lkey, ws, kAtStride, vp, w);
        *reinterpret_cast<uint4*>(row + 4 * c4) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Starts the copy of the warp's 32 decoded rows (contiguous: 32 x 256 B from
// `src`, the warp's first token) into its tile, rows kFullRow words apart
// (cp.async, one commit group).  Copy i moves rows 2i and 2i + 1, lane l the
// 16 bytes at (l & 15) * 16 of row 2i + (l >> 4), so every instruction reads
// 512 contiguous bytes.  Rows from `valid` on are zero-filled (source size 0:
// nothing is read).
__device__ __forceinline__ void stage_rows_async(uint32_t tile, const uint16_t* src, int valid, int lane)
{
    const uint16_t* p = src + (lane >> 4) * 128 + (lane & 15) * 8;
    uint32_t d = tile + (uint32_t)((lane >> 4) * kFullRow * 4 + (lane & 15) * 16);
#pragma unroll 4
    for (int r = lane >> 4; r < 32; r += 2) {
        const bool ok = r < valid;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(ok ? p : src), "r"(ok ? 16u : 0u)
                     : "memory");
        p += 2 * 128;
        d += 2 * kFullRow * 4;
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void stage_rows_wait()
{
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// S += Q . K^T over dims 32 qd .. 32 qd + 31 of the warp's 32 staged tokens;
// `stage_sh` addresses those dims of token 0, rows ROW words apart.
template <int ROW = kStageRow>
__device__ __forceinline__ void k_quarter_mma(float (&S)[4][4], const uint32_t* qrow, uint32_t stage_sh, int lane,
                                              int qd)
{
    const int j0 = qd * 16;  // dims 32 qd.. as bf16 pairs
    const uint32_t a00 = qrow[j0], a02 = qrow[j0 + 4], a10 = qrow[j0 + 8], a12 = qrow[j0 + 12];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        // matrices (lane >> 3): dims 0-7, 8-15, 16-23, 24-31 of tokens nt*8 + (lane & 7)
        uint32_t bfr[4];
        ldsm_x4(stage_sh + (uint32_t)(((nt * 8 + (lane & 7)) * ROW + (lane >> 3) * 4) * 4), bfr);
        mma_bf16(S[nt], a00, 0u, a02, 0u, bfr[0], bfr[1]);
        mma_bf16(S[nt], a10, 0u, a12, 0u, bfr[2], bfr[3]);
    }
}

// P . V over the warp's 32 staged tokens for dims 32 qd .. 32 qd + 31, written
// over those dims' columns of the warp's own tile once every lane has read
// them: head g's 32 sums go to rows 2g (dims 0-15) and 2g + 1 (dims 16-31),
// words 16 qd .. 16 qd + 15 (plain stores; no other warp touches the tile).
template <int G>
__device__ __forceinline__ void v_quarter_part(float* tile, const uint32_t (&pa)[2][4], uint32_t stage_sh, int lane,
                                               int gid, int tig, int qd)
{
    uint32_t bfr[4][4];
#pragma unroll
    for (int nd = 0; nd < 4; ++nd) ldsm_x4_t(stage_sh + (uint32_t)((lane * kFullRow + nd * 4) * 4), bfr[nd]);
    float o[4][4];
#pragma unroll
    for (int nd = 0; nd < 4; ++nd) {
#pragma unroll
        for (int e = 0; e < 4; ++e) o[nd][e] = 0.0f;
        mma_bf16(o[nd], pa[0][0], pa[0][1], pa[0][2], pa[0][3], bfr[nd][0], bfr[nd][1]);
        mma_bf16(o[nd], pa[1][0], pa[1][1], pa[1][2], pa[1][3], bfr[nd][2], bfr[nd][3]);
    }
    __syncwarp();  // the quarter's columns are read by every lane
    if (gid < G) {
#pragma unroll
        for (int nd = 0; nd < 4; ++nd) {
            const int dd = nd * 8 + 2 * tig;  // dim within the quarter
            *reinterpret_cast<float2*>(tile + (2 * gid + (dd >> 4)) * kFullRow + 16 * qd + (dd & 15)) =
                make_float2(o[nd][0] + o[nd][2], o[nd][1] + o[nd][3]);
        }
    }
}

// acc[head][dims 32 qd ..] += P . V over the warp's 32 staged tokens.
template <int G, int ROW = kStageRow>
__device__ __forceinline__ void v_quarter_mma(float* s_acc, const uint32_t (&pa)[2][4], uint32_t stage_sh, int lane,
                                              int gid, int tig, int qd)
{
#pragma unroll
    for (int nd = 0; nd < 4; ++nd) {
        // matrices (lane >> 3): tokens 0-7, 8-15, 16-23, 24-31 of dims nd*8..; lane l addresses token l
        uint32_t bfr[4];
        ldsm_x4_t(stage_sh + (uint32_t)((lane * ROW + nd * 4) * 4), bfr);
        float o[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        mma_bf16(o, pa[0][0], pa[0][1], pa[0][2], pa[0][3], bfr[0], bfr[1]);
        mma_bf16(o, pa[1][0], pa[1][1], pa[1][2], pa[1][3], bfr[2], bfr[3]);
        if (gid < G) {
            const int d = qd * 32 + nd * 8 + 2 * tig;
            atomicAdd(&s_acc[gid * 128 + d], o[0] + o[2]);
            atomicAdd(&s_acc[gid * 128 + d + 1], o[1] + o[3]);
        }
    }
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi)
{
    return f32_to_bf16_bits(lo) | (f32_to_bf16_bits(hi) << 16);
}

// STAGED = false: the CTA decodes its split's K and V blocks itself.
// STAGED = true: the split's rows were decoded into A.kx / A.vx by the block
// decoder just before (records already applied), and are read from there.
template <int G, bool STAGED>
__global__ void __launch_bounds__(STAGED ? kStTokens : kAtThreads, STAGED ? 3 : 1)
    attn_split_kernel(const __grid_constant__ AttnArgs A)
{
    constexpr int W = STAGED ? kStWarps : kAtWarps;  // warps, 32 tokens each
    constexpr int NT = W * 32;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t* smem = aligned_smem(smem_raw);
    // unstaged only: tables, stream words, nibbles, per-token exchange
    uint8_t* s_lut = smem + kOffLut;
    float* s_Ct = reinterpret_cast<float*>(smem + kOffCt);
    uint32_t* s_w = reinterpret_cast<uint32_t*>(smem + kOffWords);
    float* s_x = reinterpret_cast<float*>(smem + kOffX);
    float* s_qf = reinterpret_cast<float*>(smem + kOffQf);    // unstaged only
    float* s_acc = reinterpret_cast<float*>(smem + kOffAcc);  // unstaged only
    uint16_t* s_qb = reinterpret_cast<uint16_t*>(smem + (STAGED ? kSOffQb : kOffQb));
    float* s_red = reinterpret_cast<float*>(smem + (STAGED ? kSOffRed : kOffRed));

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;  // mma fragment coordinates
    const int split = (STAGED ? A.split0 : 0) + (int)blockIdx.x, bh = blockIdx.y;
    const int b = bh / A.H, h = bh - b * A.H;
    const int Hq = A.H * G;
    const int tok0 = split * NT + warp * 32;  // first token of this warp
    const bool have = tok0 + lane < A.S;
    const int64_t blk = (int64_t)bh * A.s_cap + tok0 + lane;

    // q of the group's heads (rows >= G are zero), accumulator cleared
    for (int i = tid; i < kHeads * 128; i += NT) {
        const int g = i >> 7, d = i & 127;
        const uint16_t v = (g < G) ? A.q[((int64_t)b * Hq + h * G + g) * 128 + d] : (uint16_t)0;
        s_qb[g * kQbRow + d] = v;
        if constexpr (!STAGED) {
            s_qf[i] = bf16_bits_to_f32(v);
            s_acc[i] = 0.0f;
        }
    }
    if constexpr (!STAGED) stage_tables<kAtThreads>(A.ktb, s_lut, s_Ct, tid);
    __syncthreads();

    uint32_t* ws = s_w + tid;
    uint32_t* nb = reinterpret_cast<uint32_t*>(smem + kOffNib) + tid;
    uint32_t* stage = reinterpret_cast<uint32_t*>(smem + kOffStage) + warp * 32 * kStageRow;  // unstaged
    uint32_t* row = stage + lane * kStageRow;
    const uint32_t stage_sh = (uint32_t)__cvta_generic_to_shared(stage);
    float* xw = s_x + warp * 32 * kHeads;
    // staged: this warp's tile of whole rows, and this lane's row in it
    const uint32_t tile_sh = (uint32_t)__cvta_generic_to_shared(smem + kSOffTile) + warp * 32 * kFullRow * 4;
    const int64_t xoff = ((int64_t)bh * A.cstride + (tok0 - A.c0)) * 128;  // the warp's first row
    const int valid = min(32, A.S - tok0);                                   // rows before the end (may be <= 0)

    // ---------------- K pass: S = Q K^T for the warp's 32 tokens
    float S[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) S[nt][e] = 0.0f;
    if constexpr (STAGED) {
        const uint32_t* qrow = reinterpret_cast<const uint32_t*>(s_qb + gid * kQbRow) + tig;
        stage_rows_async(tile_sh, valid > 0 ? A.kx + xoff : A.kx, valid, lane);
        stage_rows_wait();
        __syncwarp();
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) k_quarter_mma<kFullRow>(S, qrow, tile_sh + 64u * qd, lane, qd);
        __syncwarp();  // every lane's K reads are done: the V rows go into the same tile during the softmax
        stage_rows_async(tile_sh, valid > 0 ? A.vx + xoff : A.vx, valid, lane);
    } else {
        uint4 q0, q1, q2, q3;
        const float s = load_block(A.kblk + blk * ECCO_BLOCK_BYTES, have, q0, q1, q2, q3, A.ktb->S_t);
        stage_words(ws, kAtStride, q0, q1, q2, q3);
        const ValuePlanes vp = make_planes(s, s_Ct, (int)((q0.x >> 8) & 63u));
        const uint32_t lkey = lut_key(s_lut, (q0.x >> 8) & 255u);
        Stream st{q0.x, q0.y, kHdrBits, 2, kPayloadBits};
        // qrow[j] = q[gid][2 (tig + j)], q[gid][2 (tig + j) + 1]
        const uint32_t* qrow = reinterpret_cast<const uint32_t*>(s_qb + gid * kQbRow) + tig;
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
            decode_quarter(st, lkey, ws, vp, row, nb, qd);
            __syncwarp();
            k_quarter_mma(S, qrow, stage_sh, lane, qd);
            __syncwarp();
        }
        // outlier records: score += (new - old) * q[g][i], exchanged through shared memory
        float corr[kHeads];
#pragma unroll
        for (int g = 0; g < kHeads; ++g) corr[g] = 0.0f;
        bool any = false;
        for_records(st, ws, nb, s, vp, A.ktb->o_of_q, [&](int i, float dv) {
            any = true;
#pragma unroll
            for (int g = 0; g < G; ++g) corr[g] = fmaf(dv, s_qf[g * 128 + i], corr[g]);
        });
        if (__any_sync(0xffffffffu, any)) {
            *reinterpret_cast<float4*>(xw + lane * kHeads) = make_float4(corr[0], corr[1], corr[2], corr[3]);
            *reinterpret_cast<float4*>(xw + lane * kHeads + 4) = make_float4(corr[4], corr[5], corr[6], corr[7]);
            __syncwarp();
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                S[nt][0] += xw[(nt * 8 + 2 * tig) * kHeads + gid];
                S[nt][1] += xw[(nt * 8 + 2 * tig + 1) * kHeads + gid];
            }
            __syncwarp();
        }
    }

    // ---------------- softmax over this split's tokens (head = gid)
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const bool ok = tok0 + nt * 8 + 2 * tig + e < A.S;
            S[nt][e] = ok ? S[nt][e] * A.scale : -INFINITY;
            mx = fmaxf(mx, S[nt][e]);
        }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    if (tig == 0) s_red[warp * kHeads + gid] = mx;
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < W; ++w) M = fmaxf(M, s_red[w * kHeads + gid]);
    float sum = 0.0f;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float p = expf(S[nt][e] - M);  // exp(-inf) = 0 past the end
            S[nt][e] = p;
            sum += p;
            if constexpr (!STAGED) xw[(nt * 8 + 2 * tig + e) * kHeads + gid] = p;  // p by token, for the V records
        }
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
    if (tig == 0) s_red[W * kHeads + warp * kHeads + gid] = sum;
    __syncthreads();  // also: the K tables are no longer read
    float L = 0.0f;
#pragma unroll
    for (int w = 0; w < W; ++w) L += s_red[W * kHeads + w * kHeads + gid];
    if constexpr (!STAGED) stage_tables<kAtThreads>(A.vtb, s_lut, s_Ct, tid);

    // A fragments of P, k-step ks = tokens 16 ks + (0..15):
    // a0 / a2 (rows 0-7) = bf16(p), a1 / a3 (rows 8-15) = bf16(p - bf16(p))
    uint32_t pa[2][4];
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const float p0 = S[2 * ks + half][0], p1 = S[2 * ks + half][1];
            const uint32_t hi = pack2_bf16(p0, p1);
            const float r0 = p0 - __uint_as_float(hi << 16), r1 = p1 - __uint_as_float(hi & 0xffff0000u);
            pa[ks][2 * half] = hi;
            pa[ks][2 * half + 1] = pack2_bf16(r0, r1);
        }
    }
    if constexpr (!STAGED) __syncthreads();  // the V tables are staged

    // ---------------- V pass: O = P V, and this split's partial result
    float* out = A.ws + ((int64_t)b * Hq + h * G) * A.splits * 130;
    if constexpr (STAGED) {
        stage_rows_wait();
        __syncwarp();  // other lanes' copies landed too
        float* tiles = reinterpret_cast<float*>(smem + kSOffTile);
#pragma unroll
        for (int qd = 0; qd < 4; ++qd)
            v_quarter_part<G>(tiles + warp * 32 * kFullRow, pa, tile_sh + 64u * qd, lane, gid, tig, qd);
        __syncthreads();
        for (int i = tid; i < G * 128; i += NT) {
            const int g = i >> 7, d = i & 127, dd = d & 31;
            const float* pp = tiles + (2 * g + (dd >> 4)) * kFullRow + 16 * (d >> 5) + (dd & 15);
            float acc = 0.0f;
#pragma unroll
            for (int w = 0; w < W; ++w) acc += pp[w * 32 * kFullRow];
            out[((int64_t)g * A.splits + split) * 130 + d] = acc;
        }
    } else {
        uint4 q0, q1, q2, q3;
        const float s = load_block(A.vblk + blk * ECCO_BLOCK_BYTES, have, q0, q1, q2, q3, A.vtb->S_t);
        stage_words(ws, kAtStride, q0, q1, q2, q3);
        const ValuePlanes vp = make_planes(s, s_Ct, (int)((q0.x >> 8) & 63u));
        const uint32_t lkey = lut_key(s_lut, (q0.x >> 8) & 255u);
        Stream st{q0.x, q0.y, kHdrBits, 2, kPayloadBits};
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
            decode_quarter(st, lkey, ws, vp, row, nb, qd);
            __syncwarp();
            v_quarter_mma<G>(s_acc, pa, stage_sh, lane, gid, tig, qd);
            __syncwarp();
        }
        const float* pt = xw + lane * kHeads;  // this token's p per head
        for_records(st, ws, nb, s, vp, A.vtb->o_of_q, [&](int i, float dv) {
#pragma unroll
            for (int g = 0; g < G; ++g) atomicAdd(&s_acc[g * 128 + i], pt[g] * dv);
        });
        __syncthreads();
        for (int i = tid; i < G * 128; i += NT) {
            const int g = i >> 7, d = i & 127;
            out[((int64_t)g * A.splits + split) * 130 + d] = s_acc[i];
        }
    }
    if (warp == 0 && tig == 0 && gid < G) {
        out[((int64_t)gid * A.splits + split) * 130 + 128] = M;
        out[((int64_t)gid * A.splits + split) * 130 + 129] = L;
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

template <int G, bool STAGED>
cudaError_t configure_attn()
{
    static std::atomic<uint64_t> configured{0};
    return set_max_smem_once(configured, (const void*)attn_split_kernel<G, STAGED>,
                             STAGED ? kAttnSmemStaged : kAttnSmem);
}

template <int G>
cudaError_t run_attn(const AttnArgs& A, int B, cudaStream_t s, float* out)
{
    cudaError_t e = configure_attn<G, false>();
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)A.splits, (unsigned)(B * A.H));
    attn_split_kernel<G, false><<<grid, kAtThreads, kAttnSmem, s>>>(A);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_merge_kernel<<<B * A.H * G, 128, 0, s>>>(A.ws, A.splits, out);
    return cudaGetLastError();
}

// Staged: per chunk of tokens, the block decoder writes the chunk's K and V
// rows to the scratch (one two-segment launch), then the split kernel reads
// them; the merge runs once over all splits.
template <int G>
cudaError_t run_attn_staged(AttnArgs A, int B, const ecco_tables* kt, const ecco_tables* vt, uint16_t* scratch,
                            cudaStream_t s, float* out)
{
    cudaError_t e = configure_attn<G, true>();
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)B * A.H, C = staged_chunk_tokens(B, A.H, A.S);
    A.kx = scratch;
    A.vx = scratch + rows * C * kG;
    A.cstride = C;
    for (int64_t c0 = 0; c0 < A.S; c0 += C) {
        const int64_t cn = (A.S - c0 < C) ? A.S - c0 : C;
        ecco_segment seg[2];
        seg[0] = ecco_segment{kt, A.kblk, scratch, ecco_desc{rows, cn, A.s_cap, C, c0, 0}};
        seg[1] = ecco_segment{vt, A.vblk, scratch + rows * C * kG, ecco_desc{rows, cn, A.s_cap, C, c0, 0}};
        e = launch_decode_multi(seg, 2, s);
        if (e != cudaSuccess) return e;
        A.c0 = c0;
        A.split0 = (int)(c0 / kStTokens);
        dim3 grid((unsigned)((cn + kStTokens - 1) / kStTokens), (unsigned)rows);
        attn_split_kernel<G, true><<<grid, kStTokens, kAttnSmemStaged, s>>>(A);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    attn_merge_kernel<<<B * A.H * G, 128, 0, s>>>(A.ws, A.splits, out);
    return cudaGetLastError();
}

}  // namespace

int attention_splits(int seq_len) { return (seq_len + kAtThreads - 1) / kAtThreads; }

int attention_staged_splits(int seq_len) { return (seq_len + kStTokens - 1) / kStTokens; }

int64_t staged_chunk_tokens(int B, int H, int seq_len)
{
    const int64_t per_token = (int64_t)B * H * 2 * kG * 2;  // K and V bf16 rows of one token position
    int64_t c = kStagedScratchBytes / per_token / kAtThreads * kAtThreads;
    const int64_t whole = ((int64_t)seq_len + kAtThreads - 1) / kAtThreads * kAtThreads;
    if (c < kAtThreads) c = kAtThreads;
    return c < whole ? c : whole;
}

cudaError_t launch_attention(const ecco_tables* kt, const ecco_tables* vt, const uint8_t* kblk,
                             const uint8_t* vblk, int64_t s_cap, int B, int H, int G, int S,
                             const uint16_t* q, float scale, float* out, float* ws, cudaStream_t s)
{
    AttnArgs A{kt->d, vt->d, kblk, vblk, s_cap, H, G, S, attention_splits(S), q, scale, ws, nullptr, nullptr, 0, 0, 0};
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

cudaError_t launch_attention_staged(const ecco_tables* kt, const ecco_tables* vt, const uint8_t* kblk,
                                    const uint8_t* vblk, int64_t s_cap, int B, int H, int G, int S,
                                    const uint16_t* q, float scale, float* out, float* ws, uint16_t* scratch,
                                    cudaStream_t s)
{
    AttnArgs A{kt->d, vt->d, kblk, vblk, s_cap, H, G, S, attention_staged_splits(S), q, scale, ws,
               nullptr, nullptr, 0, 0, 0};
    switch (G) {
        case 1: return run_attn_staged<1>(A, B, kt, vt, scratch, s, out);
        case 2: return run_attn_staged<2>(A, B, kt, vt, scratch, s, out);
        case 3: return run_attn_staged<3>(A, B, kt, vt, scratch, s, out);
        case 4: return run_attn_staged<4>(A, B, kt, vt, scratch, s, out);
        case 5: return run_attn_staged<5>(A, B, kt, vt, scratch, s, out);
        case 6: return run_attn_staged<6>(A, B, kt, vt, scratch, s, out);
        case 7: return run_attn_staged<7>(A, B, kt, vt, scratch, s, out);
        case 8: return run_attn_staged<8>(A, B, kt, vt, scratch, s, out);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ecco

// ------------------------------------------------ static workspace variant
// ecco_decode_attention_static: the split partials go to this file-scope
// device array instead of a caller workspace, for callers that cannot allocate
// device memory on the attention path (a plain-C host loop without a caching
// allocator; code that must not call cudaMalloc, which can synchronize the
// device and fail under memory pressure).  Nothing in it needs to start at
// zero.  Calls that overlap on one device race on it.
static __device__ __align__(256) float g_attn_static_ws[ECCO_ATTENTION_STATIC_WS_BYTES / sizeof(float)];

static constexpr int kMaxDevices = 64;
static std::atomic<void*> g_static_ws_addr[kMaxDevices];  // per device, looked up once with that device current

extern "C" int ecco_decode_attention_static(const ecco_tables* kt, const ecco_tables* vt, const uint8_t* kblk,
                                            const uint8_t* vblk, int64_t s_cap, int batch, int kv_heads,
                                            int group, int seq_len, const uint16_t* q, float scale, float* out,
                                            void* stream)
{
    // the same checks, in the same order, as ecco_decode_attention; then the size limit
    int rc = ecco::check_attention(kt, vt, kblk, vblk, s_cap, batch, kv_heads, group, seq_len, q, out);
    if (rc) return rc;
    const size_t need = ecco_decode_attention_workspace_bytes(batch, kv_heads, group, seq_len);
    if (need > (size_t)ECCO_ATTENTION_STATIC_WS_BYTES) return ECCO_ERR_WORKSPACE;
    const int dev = kt->device;  // the current device (checked above)
    if (dev < 0 || dev >= kMaxDevices) return ECCO_ERR_UNSUPPORTED;
    void* ws = g_static_ws_addr[dev].load(std::memory_order_acquire);
    if (!ws) {
        if (cudaGetSymbolAddress(&ws, g_attn_static_ws) != cudaSuccess || !ws) return ECCO_ERR_CUDA;
        g_static_ws_addr[dev].store(ws, std::memory_order_release);
    }
    return ecco_decode_attention(kt, vt, kblk, vblk, s_cap, batch, kv_heads, group, seq_len, q, scale, out, ws,
                                 (size_t)ECCO_ATTENTION_STATIC_WS_BYTES, stream);
}
