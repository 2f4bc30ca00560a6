// Table upload: validates a table blob and derives the device-side tables.
//
// The blob holds what the review page says is learned offline per tensor
// ("Ecco: Improving Memory Bandwidth and Capacity ...", "What carries the
// argument": 64 patterns of 15 sorted centroids, 4 Huffman codebooks per
// pattern; Fig. 4 caption: the per-tensor FP8 scale factor).  Derived here:
//   - thresholds between neighbouring centroids (a value goes to the centroid
//     whose interval holds it; a value equal to a threshold goes to the lower),
//   - canonical codewords from the code lengths (ordered by length, then
//     symbol), stored in stream order (first emitted bit in bit 0),
//   - a 256-entry decode table per codebook indexed by the next 8 stream bits
//     (every codeword is at most 8 bits long: referee comment 1, Sec. 4.2).
#include <cmath>
#include <cstring>
#include <new>

#include "ecco_bucket.cuh"
#include "ecco_internal.cuh"

namespace {

using namespace ecco;

struct Blob {
    uint32_t magic, version;
    float S_t;
    uint32_t reserved;
    float C[kNPat][kNCent];
    uint8_t len[kNPat][kNBook][kNSym];
};
static_assert(sizeof(Blob) == ECCO_TABLES_BYTES, "blob layout");

bool blob_valid(const Blob& b)
{
    if (b.magic != ECCO_TABLES_MAGIC || b.version != 1u) return false;
    if (!std::isfinite(b.S_t) || !(b.S_t >= std::ldexp(1.0f, -60)) || !(b.S_t <= std::ldexp(1.0f, 60)))
        return false;
    for (int p = 0; p < kNPat; ++p)
        for (int j = 0; j < kNCent; ++j) {
            float c = b.C[p][j];
            if (!std::isfinite(c) || std::fabs(c) > 4.0f) return false;
            if (j && !(b.C[p][j - 1] < c)) return false;
        }
    for (int p = 0; p < kNPat; ++p)
        for (int h = 0; h < kNBook; ++h) {
            unsigned space = 0;  // in units of 2^-kLMax
            for (int s = 0; s < kNSym; ++s) {
                unsigned l = b.len[p][h][s];
                if (l < 1 || l > (unsigned)kLMax) return false;
                space += 1u << (kLMax - l);
            }
            if (space != (1u << kLMax)) return false;  // complete code
        }
    return true;
}

uint32_t reverse_bits(uint32_t v, int n)
{
    uint32_t r = 0;
    for (int i = 0; i < n; ++i) r |= ((v >> i) & 1u) << (n - 1 - i);
    return r;
}

// Canonical code values from per-length counts, the construction of RFC 1951
// section 3.2.2: the first code of length l is (first code of length l-1 +
// number of codes of length l-1) << 1, and codes of one length are handed out
// in symbol order.
void canonical(const uint8_t len[kNSym], uint32_t code[kNSym])
{
    uint32_t count[kLMax + 1] = {0};
    for (int s = 0; s < kNSym; ++s) count[len[s]]++;
    uint32_t next[kLMax + 1] = {0};
    for (int l = 2; l <= kLMax; ++l) next[l] = (next[l - 1] + count[l - 1]) << 1;
    for (int s = 0; s < kNSym; ++s) code[s] = next[len[s]]++;
}

void derive(const Blob& b, DevTables* t)
{
    std::memset(t, 0, sizeof *t);
    t->S_t = b.S_t;
    const float inf = INFINITY;
    for (int p = 0; p < kNPat; ++p) {
        for (int j = 0; j < kNCent - 1; ++j) {
            float sum = b.C[p][j] + b.C[p][j + 1];  // rounded on its own (no contraction)
            t->T16[p][j] = sum * 0.5f;
        }
        t->T16[p][14] = inf;
        t->T16[p][15] = inf;
        for (int j = 0; j < kNCent; ++j) t->Ct[j][p] = b.C[p][j];
        t->Ct[15][p] = 1.0f;
        t->ends[p] = make_float2(b.C[p][0], b.C[p][kNCent - 1]);
        for (int s = 0; s < kNSym; ++s) {
            uint32_t v = 0;
            for (int h = 0; h < kNBook; ++h) v |= (uint32_t)b.len[p][h][s] << (8 * h);
            t->lens4[p][s] = v;
        }
        for (int h = 0; h < kNBook; ++h) {
            uint32_t code[kNSym];
            canonical(b.len[p][h], code);
            const uint32_t tix = (uint32_t)(h * kNPat + p);
            uint8_t one[256];  // next 8 stream bits -> symbol | length << 4, unswizzled
            for (int s = 0; s < kNSym; ++s) {
                int l = b.len[p][h][s];
                uint32_t rev = reverse_bits(code[s], l);
                t->code[p][h][s] = rev | ((uint32_t)l << 8);
                for (uint32_t tail = 0; tail < (1u << (8 - l)); ++tail) one[rev | (tail << l)] = (uint8_t)(s | (l << 4));
            }
            for (uint32_t e = 0; e < 256; ++e) t->lut[tix][e ^ ((tix & 31u) << 2)] = one[e];
        }
    }
}

// One thread per bf16 magnitude (32768) and per scale code (256).
__global__ void scale_tables_kernel(DevTables* t)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    const float S_t = t->S_t;
    if (i < 32768) {
        float r = __fdiv_rn(__uint_as_float((uint32_t)i << 16), S_t);
        t->code_of_mag[i] = (uint8_t)__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E4M3);
    }
    if (i < 256) {
        float s = 0.0f, inv = 0.0f;
        if (!scale_code_is_null((uint32_t)i)) {
            s = __fmul_rn(S_t, e4m3_to_f32((uint32_t)i));
            inv = __frcp_rn(s);
        }
        t->s_of_code[i] = s;
        t->inv_of_code[i] = inv;
        t->o_of_q[i] = __fdiv_rn((float)(int8_t)(uint8_t)i, 127.0f);
    }
}

// One thread per pattern: the map T[0] -> 0.01, T[13] -> 0.99 (before the
// scaling by 255) and the per-bucket counts of thresholds below.  A pattern
// whose map is not finite, or with two thresholds in one bucket, is marked
// for bisection.
__global__ void bucket_tables_kernel(DevTables* t)
{
    const int p = threadIdx.x;
    if (p >= kNPat) return;
    const float* T = t->T16[p];
    const float a = __fdiv_rn(0.98f, __fsub_rn(T[kNCent - 2], T[0]));
    const float b = __fsub_rn(0.01f, __fmul_rn(T[0], a));
    bool dense = !(isfinite(a) && isfinite(b) && a > 0.0f);
    uint32_t nb[kNCent - 1];
    for (int k = 0; k < kNCent - 1; ++k) {
        nb[k] = threshold_bucket(T[k], a, b);
        if (k && nb[k] <= nb[k - 1]) dense = true;
    }
    for (uint32_t n = 0; n < 256; ++n) {
        uint32_t lo = 0;
        for (int k = 0; k < kNCent - 1; ++k) lo += (nb[k] < n) ? 1u : 0u;
        t->qlo[p][n] = (uint8_t)lo;
    }
    t->qmap[p] = make_float4(a, b, dense ? 1.0f : 0.0f, 0.0f);
}

}  // namespace

extern "C" int ecco_tables_create(const void* blob, size_t nbytes, ecco_tables** out)
{
    if (!blob || !out) return ECCO_ERR_ARG;
    *out = nullptr;
    if (nbytes != ECCO_TABLES_BYTES) return ECCO_ERR_TABLES;
    Blob b;
    std::memcpy(&b, blob, sizeof b);
    if (!blob_valid(b)) return ECCO_ERR_TABLES;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ECCO_ERR_CUDA;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return ECCO_ERR_CUDA;
    if (prop.major != 10) return ECCO_ERR_UNSUPPORTED;

    timeout_flag();  // the tensor-core pipeline's timeout flag, allocated once, off the hot path
    DevTables* host = new (std::nothrow) DevTables;
    if (!host) return ECCO_ERR_ARG;
    derive(b, host);
    DevTables* d = nullptr;
    if (cudaMalloc(&d, sizeof(DevTables)) != cudaSuccess) {
        delete host;
        return ECCO_ERR_CUDA;
    }
    cudaError_t e = cudaMemcpy(d, host, sizeof(DevTables), cudaMemcpyHostToDevice);
    delete host;
    if (e == cudaSuccess) {
        scale_tables_kernel<<<32768 / 256, 256>>>(d);
        bucket_tables_kernel<<<1, kNPat>>>(d);
        e = cudaGetLastError();
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
    }
    if (e != cudaSuccess) {
        cudaFree(d);
        return ECCO_ERR_CUDA;
    }
    ecco_tables* t = new (std::nothrow) ecco_tables;
    if (!t) {
        cudaFree(d);
        return ECCO_ERR_ARG;
    }
    t->device = dev;
    t->d = d;
    *out = t;
    return ECCO_OK;
}

extern "C" int ecco_tables_destroy(ecco_tables* t)
{
    if (!t) return ECCO_ERR_ARG;
    int cur = 0;
    cudaGetDevice(&cur);
    if (cur != t->device) cudaSetDevice(t->device);
    cudaError_t e = cudaFree(t->d);
    if (cur != t->device) cudaSetDevice(cur);
    delete t;
    return e == cudaSuccess ? ECCO_OK : ECCO_ERR_CUDA;
}
