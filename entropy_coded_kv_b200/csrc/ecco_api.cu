// C ABI entry points: argument validation, device checks, dispatch to the
// kernel launchers.  Nothing here allocates device memory.
#include <cmath>
#include <cstdint>

#include "ecco_internal.cuh"

namespace ecco {

// SM count of the current device, looked up once per device (safe from
// several host threads: each slot is written with the same value).
int device_sm_count()
{
    static std::atomic<int> cached[kMaxDeviceBits];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    const bool slot = dev >= 0 && dev < kMaxDeviceBits;
    int sms = slot ? cached[dev].load(std::memory_order_relaxed) : 0;
    if (sms > 0) return sms;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 1;
    if (slot) cached[dev].store(sms, std::memory_order_relaxed);
    return sms;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_tables(const ecco_tables* t)
{
    if (!t || !t->d) return ECCO_ERR_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return ECCO_ERR_CUDA;
    if (dev != t->device) return ECCO_ERR_DEVICE;
    return ECCO_OK;
}

int check_desc(const ecco_desc& d)
{
    if (d.rows < 0 || d.groups_per_row < 0 || d.src_row_stride < 0 || d.dst_row_stride < 0 ||
        d.src_offset < 0 || d.dst_offset < 0)
        return ECCO_ERR_ARG;
    if (d.rows > 1 && d.dst_row_stride < d.groups_per_row) return ECCO_ERR_ARG;
    // keep every group index representable: offset + (rows-1)*stride + gpr < 2^40
    const int64_t lim = (int64_t)1 << 40;
    if (d.rows > lim || d.groups_per_row > lim) return ECCO_ERR_ARG;
    if (d.rows > 0 && d.groups_per_row > 0) {
        // at most 2^31 - 2048 groups per tensor and call (512 GiB of bf16):
        // the kernels index a tensor's groups with 32-bit integers
        if (d.rows > (((int64_t)1 << 31) - 2048) / d.groups_per_row) return ECCO_ERR_ARG;
        if (d.src_row_stride > lim / (d.rows > 1 ? d.rows : 1)) return ECCO_ERR_ARG;
        if (d.dst_row_stride > lim / (d.rows > 1 ? d.rows : 1)) return ECCO_ERR_ARG;
        if (d.src_offset > lim || d.dst_offset > lim) return ECCO_ERR_ARG;
    }
    return ECCO_OK;
}

int status(cudaError_t e) { return e == cudaSuccess ? ECCO_OK : ECCO_ERR_CUDA; }

}  // namespace
}  // namespace ecco

using namespace ecco;

extern "C" int ecco_select_encode(const ecco_tables* t, const uint16_t* x, ecco_desc d,
                                  uint8_t* blocks, ecco_stats* stats, void* stream)
{
    int rc = check_tables(t);
    if (rc) return rc;
    if ((rc = check_desc(d))) return rc;
    if (d.rows == 0 || d.groups_per_row == 0) return ECCO_OK;
    if (!x || !blocks) return ECCO_ERR_ARG;
    if (!aligned16(x) || !aligned16(blocks) || (stats && (reinterpret_cast<uintptr_t>(stats) & 7u)))
        return ECCO_ERR_ALIGN;
    return status(launch_encode(t, x, d, blocks, stats, (cudaStream_t)stream));
}

extern "C" int ecco_select_encode_ex(const ecco_tables* t, const uint16_t* x, ecco_desc d, uint8_t* blocks,
                                     ecco_stats* stats, int select, int n_patterns, void* stream)
{
    if (select != ECCO_SELECT_MINMAX && select != ECCO_SELECT_MSE) return ECCO_ERR_ARG;
    if (n_patterns < 1 || n_patterns > ECCO_NPAT) return ECCO_ERR_ARG;
    int rc = check_tables(t);
    if (rc) return rc;
    if ((rc = check_desc(d))) return rc;
    if (d.rows == 0 || d.groups_per_row == 0) return ECCO_OK;
    if (!x || !blocks) return ECCO_ERR_ARG;
    if (!aligned16(x) || !aligned16(blocks) || (stats && (reinterpret_cast<uintptr_t>(stats) & 7u)))
        return ECCO_ERR_ALIGN;
    return status(launch_encode(t, x, d, blocks, stats, (cudaStream_t)stream, select, n_patterns));
}

extern "C" int ecco_select_encode_act(const ecco_tables* t, const uint16_t* x, ecco_desc d, uint8_t* blocks,
                                      ecco_stats* stats, void* stream)
{
    int rc = check_tables(t);
    if (rc) return rc;
    if ((rc = check_desc(d))) return rc;
    if (d.rows == 0 || d.groups_per_row == 0) return ECCO_OK;
    if (!x || !blocks) return ECCO_ERR_ARG;
    if (!aligned16(x) || !aligned16(blocks) || (stats && (reinterpret_cast<uintptr_t>(stats) & 7u)))
        return ECCO_ERR_ALIGN;
    return status(launch_encode_act(t, x, d, blocks, stats, (cudaStream_t)stream));
}

extern "C" int ecco_decode_act(const ecco_tables* t, const uint8_t* blocks, ecco_desc d, uint16_t* y,
                               void* stream)
{
    int rc = check_tables(t);
    if (rc) return rc;
    if ((rc = check_desc(d))) return rc;
    if (d.rows == 0 || d.groups_per_row == 0) return ECCO_OK;
    if (!blocks || !y) return ECCO_ERR_ARG;
    if (!aligned16(blocks) || !aligned16(y)) return ECCO_ERR_ALIGN;
    return status(launch_decode_act(t, blocks, d, y, (cudaStream_t)stream));
}

extern "C" int ecco_decode(const ecco_tables* t, const uint8_t* blocks, ecco_desc d, uint16_t* y,
                           void* stream)
{
    int rc = check_tables(t);
    if (rc) return rc;
    if ((rc = check_desc(d))) return rc;
    if (d.rows == 0 || d.groups_per_row == 0) return ECCO_OK;
    if (!blocks || !y) return ECCO_ERR_ARG;
    if (!aligned16(blocks) || !aligned16(y)) return ECCO_ERR_ALIGN;
    return status(launch_decode(t, blocks, d, y, (cudaStream_t)stream));
}

extern "C" int ecco_decode_speculative(const ecco_tables* t, const uint8_t* blocks, ecco_desc d, uint16_t* y,
                                       void* stream)
{
    int rc = check_tables(t);
    if (rc) return rc;
    if ((rc = check_desc(d))) return rc;
    if (d.rows == 0 || d.groups_per_row == 0) return ECCO_OK;
    if (!blocks || !y) return ECCO_ERR_ARG;
    if (!aligned16(blocks) || !aligned16(y)) return ECCO_ERR_ALIGN;
    return status(launch_decode_spec(t, blocks, d, y, (cudaStream_t)stream));
}

extern "C" int ecco_decode_gemv(const ecco_tables* t, const uint8_t* blocks, int64_t rows,
                                int64_t cols, const uint16_t* x, int batch, float* y, void* stream)
{
    int rc = check_tables(t);
    if (rc) return rc;
    if (rows < 0 || cols < 0 || (cols % ECCO_GROUP) != 0 || batch < 1 || batch > 16)
        return ECCO_ERR_ARG;
    if (rows > ((int64_t)1 << 34) || cols > ((int64_t)1 << 34)) return ECCO_ERR_ARG;
    if (rows == 0) return ECCO_OK;
    if (!y) return ECCO_ERR_ARG;
    if (cols == 0) return status(cudaMemsetAsync(y, 0, sizeof(float) * (size_t)batch * (size_t)rows,
                                                 (cudaStream_t)stream));
    if (!blocks || !x) return ECCO_ERR_ARG;
    if (!aligned16(blocks) || !aligned16(x) || !aligned16(y)) return ECCO_ERR_ALIGN;
    if (batch > 4 && timeout_raised()) return ECCO_ERR_TIMEOUT;  // an earlier tensor-core launch gave up
    return status(launch_gemv(t, blocks, rows, cols, x, batch, y, (cudaStream_t)stream));
}

extern "C" int ecco_decode_multi(const ecco_segment* segs, int n, void* stream)
{
    if (n < 0 || n > ECCO_MAX_SEGMENTS || (n > 0 && !segs)) return ECCO_ERR_ARG;
    for (int i = 0; i < n; ++i) {
        int rc = check_tables(segs[i].tables);
        if (rc) return rc;
        if ((rc = check_desc(segs[i].desc))) return rc;
        if (segs[i].desc.rows == 0 || segs[i].desc.groups_per_row == 0) continue;
        if (!segs[i].src || !segs[i].dst) return ECCO_ERR_ARG;
        if (!aligned16(segs[i].src) || !aligned16(segs[i].dst)) return ECCO_ERR_ALIGN;
    }
    return status(launch_decode_multi(segs, n, (cudaStream_t)stream));
}

extern "C" int ecco_encode_multi(const ecco_segment* segs, int n, ecco_stats* stats, void* stream)
{
    if (n < 0 || n > ECCO_MAX_SEGMENTS || (n > 0 && !segs)) return ECCO_ERR_ARG;
    if (stats && (reinterpret_cast<uintptr_t>(stats) & 7u)) return ECCO_ERR_ALIGN;
    for (int i = 0; i < n; ++i) {
        int rc = check_tables(segs[i].tables);
        if (rc) return rc;
        if ((rc = check_desc(segs[i].desc))) return rc;
        if (segs[i].desc.rows == 0 || segs[i].desc.groups_per_row == 0) continue;
        if (!segs[i].src || !segs[i].dst) return ECCO_ERR_ARG;
        if (!aligned16(segs[i].src) || !aligned16(segs[i].dst)) return ECCO_ERR_ALIGN;
    }
    return status(launch_encode_multi(segs, n, stats, (cudaStream_t)stream));
}

extern "C" size_t ecco_decode_attention_workspace_bytes(int batch, int kv_heads, int group, int seq_len)
{
    if (batch < 1 || kv_heads < 1 || group < 1 || group > 8 || seq_len < 1) return 0;
    return sizeof(float) * 130 * (size_t)batch * (size_t)kv_heads * (size_t)group *
           (size_t)attention_splits(seq_len);
}

namespace ecco {
// Checks shared by the attention entry points, in the order the header states:
// tables, sizes, pointers, then alignment of the inputs and the output.
int check_attention(const ecco_tables* kt, const ecco_tables* vt, const uint8_t* kblk, const uint8_t* vblk,
                    int64_t s_cap, int batch, int kv_heads, int group, int seq_len, const uint16_t* q,
                    const float* out)
{
    int rc = check_tables(kt);
    if (rc) return rc;
    if ((rc = check_tables(vt))) return rc;
    if (batch < 1 || kv_heads < 1 || group < 1 || group > 8 || seq_len < 1 || s_cap < seq_len)
        return ECCO_ERR_ARG;
    if ((int64_t)batch * kv_heads > 65535 || s_cap > ((int64_t)1 << 34)) return ECCO_ERR_ARG;
    if (!kblk || !vblk || !q || !out) return ECCO_ERR_ARG;
    if (!aligned16(kblk) || !aligned16(vblk) || (reinterpret_cast<uintptr_t>(q) & 1u) ||
        (reinterpret_cast<uintptr_t>(out) & 3u))
        return ECCO_ERR_ALIGN;
    return ECCO_OK;
}
}  // namespace ecco

extern "C" int ecco_decode_attention(const ecco_tables* kt, const ecco_tables* vt, const uint8_t* kblk,
                                     const uint8_t* vblk, int64_t s_cap, int batch, int kv_heads,
                                     int group, int seq_len, const uint16_t* q, float scale, float* out,
                                     void* ws, size_t ws_bytes, void* stream)
{
    int rc = check_attention(kt, vt, kblk, vblk, s_cap, batch, kv_heads, group, seq_len, q, out);
    if (rc) return rc;
    if (!ws) return ECCO_ERR_ARG;
    if (ws_bytes < ecco_decode_attention_workspace_bytes(batch, kv_heads, group, seq_len)) return ECCO_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(ws) & 3u) return ECCO_ERR_ALIGN;
    return status(launch_attention(kt, vt, kblk, vblk, s_cap, batch, kv_heads, group, seq_len, q, scale,
                                   out, static_cast<float*>(ws), (cudaStream_t)stream));
}

namespace {
constexpr size_t kScratchAlign = 256;
size_t staged_partials_bytes(int batch, int kv_heads, int group, int seq_len)
{
    if (ecco_decode_attention_workspace_bytes(batch, kv_heads, group, seq_len) == 0) return 0;
    const size_t p = sizeof(float) * 130 * (size_t)batch * (size_t)kv_heads * (size_t)group *
                     (size_t)ecco::attention_staged_splits(seq_len);
    return (p + kScratchAlign - 1) / kScratchAlign * kScratchAlign;
}
}  // namespace

extern "C" size_t ecco_decode_attention_staged_workspace_bytes(int batch, int kv_heads, int group, int seq_len)
{
    if (ecco_decode_attention_workspace_bytes(batch, kv_heads, group, seq_len) == 0) return 0;
    const size_t chunk = (size_t)ecco::staged_chunk_tokens(batch, kv_heads, seq_len);
    return staged_partials_bytes(batch, kv_heads, group, seq_len) + kScratchAlign +
           2 * (size_t)batch * (size_t)kv_heads * chunk * 128 * sizeof(uint16_t);
}

extern "C" int ecco_decode_attention_staged(const ecco_tables* kt, const ecco_tables* vt, const uint8_t* kblk,
                                            const uint8_t* vblk, int64_t s_cap, int batch, int kv_heads,
                                            int group, int seq_len, const uint16_t* q, float scale, float* out,
                                            void* ws, size_t ws_bytes, void* stream)
{
    int rc = check_attention(kt, vt, kblk, vblk, s_cap, batch, kv_heads, group, seq_len, q, out);
    if (rc) return rc;
    if (!ws) return ECCO_ERR_ARG;
    if (ws_bytes < ecco_decode_attention_staged_workspace_bytes(batch, kv_heads, group, seq_len))
        return ECCO_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(ws) & 3u) return ECCO_ERR_ALIGN;
    // partials first, then the decoded-row scratch from the next 256-byte boundary
    const uintptr_t sc = (reinterpret_cast<uintptr_t>(ws) + staged_partials_bytes(batch, kv_heads, group, seq_len) +
                          kScratchAlign - 1) / kScratchAlign * kScratchAlign;
    return status(launch_attention_staged(kt, vt, kblk, vblk, s_cap, batch, kv_heads, group, seq_len, q, scale,
                                          out, static_cast<float*>(ws), reinterpret_cast<uint16_t*>(sc),
                                          (cudaStream_t)stream));
}

extern "C" int ecco_learn_tables(const uint16_t* x, int64_t n_groups, int group, int n_patterns, uint64_t seed,
                                 void* blob, size_t blob_bytes, void* stream)
{
    if (!x || !blob || blob_bytes < ECCO_TABLES_BYTES) return ECCO_ERR_ARG;
    if (n_groups < 1 || n_groups > ((int64_t)1 << 34)) return ECCO_ERR_ARG;
    if (group != ECCO_GROUP && group != ECCO_GROUP_ACT) return ECCO_ERR_ARG;
    if (n_patterns < 1 || n_patterns > ECCO_NPAT) return ECCO_ERR_ARG;
    if (!aligned16(x)) return ECCO_ERR_ALIGN;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ECCO_ERR_CUDA;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return ECCO_ERR_CUDA;
    if (prop.major != 10) return ECCO_ERR_UNSUPPORTED;
    return status(learn_tables(x, n_groups, group, n_patterns, seed, static_cast<uint8_t*>(blob),
                               (cudaStream_t)stream));
}

extern "C" int ecco_huffman_lengths(const double* w, int n, int max_len, uint8_t* lens)
{
    if (!w || !lens || n < 1 || max_len < 1 || max_len > 30) return ECCO_ERR_ARG;
    if (n > 1 && (int64_t)n > ((int64_t)1 << max_len)) return ECCO_ERR_ARG;
    for (int i = 0; i < n; ++i)
        if (!(w[i] > 0.0) || !std::isfinite(w[i])) return ECCO_ERR_ARG;
    return huffman_lengths(w, n, max_len, lens) == 0 ? ECCO_OK : ECCO_ERR_ARG;
}

extern "C" const char* ecco_strerror(int code)
{
    switch (code) {
        case ECCO_OK: return "ok";
        case ECCO_ERR_ARG: return "invalid argument";
        case ECCO_ERR_ALIGN: return "pointer not aligned as required";
        case ECCO_ERR_TABLES: return "invalid table blob";
        case ECCO_ERR_CUDA: return "CUDA runtime error";
        case ECCO_ERR_DEVICE: return "current device is not the tables' device";
        case ECCO_ERR_UNSUPPORTED: return "device is not sm_100";
        case ECCO_ERR_WORKSPACE: return "request needs more than the static attention workspace";
        case ECCO_ERR_TIMEOUT: return "a bounded device wait gave up in an earlier tensor-core launch";
        default: return "unknown error";
    }
}

extern "C" int ecco_abi_version(void) { return 1; }

extern "C" int ecco_selftest_wait_timeout(void* stream)
{
    if (!timeout_flag()) return ECCO_ERR_CUDA;
    return status(launch_wait_timeout_selftest((cudaStream_t)stream));
}
