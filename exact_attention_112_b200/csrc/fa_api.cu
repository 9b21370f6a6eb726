// fa_api.cu -- the C ABI of libfa.so (declared in include/fa.h): argument
// validation, TMA tensor-map construction, the per-device error word and the
// launches.  No device memory is allocated here.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "fa.h"
#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait

// One error word per device; kernels latch a code into it, fa_device_status()
// reads and clears it.
__device__ int g_fa_error_word;

std::mutex g_mu;
int *g_err_ptr[kMaxDevices] = {};
int g_cc_major[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int current_device(int *dev) {
    if (cudaGetDevice(dev) != cudaSuccess) return FA_ERR_CUDA;
    if (*dev < 0 || *dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    return FA_OK;
}

// Per-device set-up, done once: the error word's device address, the
// compute capability and the SM count (the persistent grid size).
int device_setup(int dev, int **err_ptr, int *sm_count = nullptr) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_err_ptr[dev]) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return FA_ERR_CUDA;
        g_cc_major[dev] = prop.major;
        g_sm_count[dev] = prop.multiProcessorCount;
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_fa_error_word) != cudaSuccess) return FA_ERR_CUDA;
        g_err_ptr[dev] = static_cast<int *>(ptr);
    }
    if (g_cc_major[dev] != 10) return FA_ERR_UNSUPPORTED;
    *err_ptr = g_err_ptr[dev];
    if (sm_count) *sm_count = g_sm_count[dev] > 0 ? g_sm_count[dev] : 1;
    return FA_OK;
}

// Persistent grid: one CTA per SM, or fewer when there are fewer units.
int persistent_grid(long long units, int sm_count) {
    return static_cast<int>(units < sm_count ? units : sm_count);
}

int get_encoder(PFN_cuTensorMapEncodeTiled_v12000 *fn) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_encode) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || p == nullptr)
            return FA_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    *fn = g_encode;
    return FA_OK;
}

// 3-D map over a [B*H, N, D] tensor of 16-bit (or, with fp8, 8-bit) values:
// box = one 128-byte row segment (64 or 128 values) x box_rows rows, 128-byte
// swizzle (matches the MMA operand layout); rows past N read as 0 and are not
// written by stores.
int make_map(CUtensorMap *m, const void *ptr, bool bf16, int D, int N, long long BH, int box_rows,
             bool fp8 = false) {
    PFN_cuTensorMapEncodeTiled_v12000 enc;
    int st = get_encoder(&enc);
    if (st != FA_OK) return st;
    const cuuint64_t elem = fp8 ? 1 : 2;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * elem, static_cast<cuuint64_t>(N) * D * elem};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elem), static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType dt = fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                       : (bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    CUresult r = enc(m, dt, 3,
                     const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shared shape/scalar validation of forward and backward.
int check_common(int B, int H, int Nq, int Nk, int D, int causal, float scale, int dtype) {
    if (B < 1 || H < 1 || Nq < 0 || Nk < 0) return FA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (dtype != FA_F16 && dtype != FA_BF16) return FA_ERR_UNSUPPORTED;
    if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
    // every index the kernels form must fit in 32-bit signed arithmetic
    const long long BH = static_cast<long long>(B) * H;
    const long long units = BH * ((static_cast<long long>(Nq) + 255) / 256);
    if (BH > INT32_MAX || units > INT32_MAX || BH * Nq > INT32_MAX) return FA_ERR_INVALID_ARG;
    if (Nq > (1 << 30) || Nk > (1 << 30)) return FA_ERR_INVALID_ARG;
    return FA_OK;
}

std::atomic<unsigned long long> g_launches{0};

struct ProfRecord {
    const char *name;
    cudaEvent_t start, stop;
};
thread_local bool t_prof_on = false;
thread_local std::vector<ProfRecord> t_prof;

}  // namespace

void fa::note_launch(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

void fa::prof_begin(cudaStream_t stream, const char *name) {
    if (!t_prof_on) return;
    ProfRecord r{name, nullptr, nullptr};
    if (cudaEventCreate(&r.start) != cudaSuccess) return;
    if (cudaEventCreate(&r.stop) != cudaSuccess) {
        cudaEventDestroy(r.start);
        return;
    }
    cudaEventRecord(r.start, stream);
    t_prof.push_back(r);
}

void fa::prof_end(cudaStream_t stream) {
    if (!t_prof_on || t_prof.empty()) return;
    cudaEventRecord(t_prof.back().stop, stream);
}

extern "C" {

unsigned long long fa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int fa_profile_enable(int on) {
    t_prof_on = on != 0;
    return FA_OK;
}

int fa_profile_read(float *ms, const char **names, int capacity, int *count) {
    if (capacity < 0 || (capacity > 0 && !ms) || !count) return FA_ERR_INVALID_ARG;
    int n = 0;
    int st = FA_OK;
    for (ProfRecord &r : t_prof) {
        float t = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess)
            st = FA_ERR_CUDA;
        if (n < capacity) {
            ms[n] = t;
            if (names) names[n] = r.name;
            ++n;
        }
        cudaEventDestroy(r.start);
        cudaEventDestroy(r.stop);
    }
    t_prof.clear();
    *count = n;
    return st;
}

const char *fa_status_string(int status) {
    switch (status) {
        case FA_OK: return "FA_OK";
        case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: invalid argument";
        case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: unsupported head dim, dtype or device";
        case FA_ERR_CUDA: return "FA_ERR_CUDA: a CUDA call failed";
        case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT: a device-side wait gave up";
        case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE: backward workspace missing or too small";
        case FA_ERR_INTERNAL: return "FA_ERR_INTERNAL: a kernel's layout self-check failed";
        default: return "unknown fa_status";
    }
}

}  // extern "C"

namespace {
// Forward parameters shared by the forward entry points (one split).
fa::FwdParams fwd_params(int B, int H, int Nq, int Nk, float scale, const float *key_bias, void *o,
                         float *lse, int *err) {
    fa::FwdParams p{};
    p.B = B;
    p.H = H;
    p.Nq = Nq;
    p.Nk = Nk;
    p.n_mblocks = (Nq + 255) / 256;
    p.n_units = p.n_mblocks * B * H;
    p.causal_off = Nk - Nq;
    p.qk_scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634074);
    p.o_scale = 1.f;
    p.bias = key_bias;
    p.o = o;
    p.lse = lse;
    p.err = err;
    p.timeout_ns = kDefaultTimeoutNs;
    p.num_splits = 1;
    p.tiles_per_split = 0;
    p.cu_q = p.cu_k = nullptr;
    p.total_q = p.total_k = 0;
    p.mask = nullptr;
    p.mask_B = p.mask_H = 1;
    p.ldm = 0;
    p.tile_flags = nullptr;
    return p;
}
}  // namespace

extern "C" {

int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int Nq,
           int Nk, int D, int causal, float scale, int dtype, const float *key_bias, void *stream) {
    int st = check_common(B, H, Nq, Nk, D, causal, scale, dtype);
    if (st != FA_OK) return st;
    if (Nq == 0) return FA_OK;
    if (!q || !o || !lse || (Nk > 0 && (!k || !v))) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
        (key_bias && !aligned16(key_bias)))
        return FA_ERR_INVALID_ARG;
    int dev;
    if ((st = current_device(&dev)) != FA_OK) return st;
    int *err = nullptr, sms = 1;
    if ((st = device_setup(dev, &err, &sms)) != FA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == FA_BF16;
    const long long BH = static_cast<long long>(B) * H;
    if (Nk == 0) {
        return fa::launch_fwd_empty(o, lse, static_cast<size_t>(BH) * Nq, D, bf16, s) == cudaSuccess
                   ? FA_OK : FA_ERR_CUDA;
    }
    fa::FwdTensorMaps tm;
    if ((st = make_map(&tm.q, q, bf16, D, Nq, BH, 128)) != FA_OK) return st;
    if ((st = make_map(&tm.k, k, bf16, D, Nk, BH, 128)) != FA_OK) return st;
    if ((st = make_map(&tm.v, v, bf16, D, Nk, BH, 128)) != FA_OK) return st;
    fa::FwdParams p = fwd_params(B, H, Nq, Nk, scale, key_bias, o, lse, err);
    cudaError_t e = fa::launch_fwd(tm, p, D, bf16 ? fa::kElemBF16 : fa::kElemF16, causal != 0,
                                   key_bias != nullptr, persistent_grid(p.n_units, sms), s);
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_fwd_fp8(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H,
               int Nq, int Nk, int D, int causal, float scale, float q_descale, float k_descale,
               float v_descale, const float *key_bias, void *stream) {
    int st = check_common(B, H, Nq, Nk, D, causal, scale, FA_BF16);
    if (st != FA_OK) return st;
    if (D != 128) return FA_ERR_UNSUPPORTED;
    for (float d : {q_descale, k_descale, v_descale})
        if (!std::isfinite(d) || !(d > 0.f)) return FA_ERR_INVALID_ARG;
    const double qk = static_cast<double>(scale) * q_descale * k_descale;
    if (!std::isfinite(qk) || qk <= 0.0 || qk > 3.0e38) return FA_ERR_INVALID_ARG;
    if (Nq == 0) return FA_OK;
    if (!q || !o || !lse || (Nk > 0 && (!k || !v))) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
        (key_bias && !aligned16(key_bias)))
        return FA_ERR_INVALID_ARG;
    int dev;
    if ((st = current_device(&dev)) != FA_OK) return st;
    int *err = nullptr, sms = 1;
    if ((st = device_setup(dev, &err, &sms)) != FA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const long long BH = static_cast<long long>(B) * H;
    if (Nk == 0) {
        return fa::launch_fwd_empty(o, lse, static_cast<size_t>(BH) * Nq, D, true, s) == cudaSuccess
                   ? FA_OK : FA_ERR_CUDA;
    }
    fa::FwdTensorMaps tm;
    if ((st = make_map(&tm.q, q, false, D, Nq, BH, 128, true)) != FA_OK) return st;
    if ((st = make_map(&tm.k, k, false, D, Nk, BH, 128, true)) != FA_OK) return st;
    if ((st = make_map(&tm.v, v, false, D, Nk, BH, 128, true)) != FA_OK) return st;
    fa::FwdParams p = fwd_params(B, H, Nq, Nk, scale, key_bias, o, lse, err);
    p.qk_scale_log2 = static_cast<float>(qk * 1.4426950408889634074);
    p.o_scale = v_descale;
    cudaError_t e = fa::launch_fwd(tm, p, D, fa::kElemE4M3, causal != 0, key_bias != nullptr,
                                   persistent_grid(p.n_units, sms), s);
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"

namespace {
// Argument checks of the general mask (see fa_fwd_mask in fa.h).
int check_mask(const float *mask, int B, int H, int Nq, int Nk, int mask_B, int mask_H, long long ldm) {
    if (!mask || !aligned16(mask)) return FA_ERR_INVALID_ARG;
    if ((mask_B != 1 && mask_B != B) || (mask_H != 1 && mask_H != H)) return FA_ERR_INVALID_ARG;
    if (ldm < Nk || ldm < 4 || ldm % 4 != 0) return FA_ERR_INVALID_ARG;
    const double elems = static_cast<double>(mask_B) * mask_H * Nq * static_cast<double>(ldm);
    if (elems > 9.0e18) return FA_ERR_INVALID_ARG;
    return FA_OK;
}
}  // namespace

extern "C" {

size_t fa_mask_tile_flags_bytes(int mask_B, int mask_H, int Nq, int Nk) {
    if (mask_B < 1 || mask_H < 1 || Nq < 0 || Nk < 0) return 0;
    return static_cast<size_t>(mask_B) * mask_H * ((static_cast<size_t>(Nq) + 127) / 128) *
           ((static_cast<size_t>(Nk) + 127) / 128);
}

int fa_mask_tile_flags(const float *mask, int mask_B, int mask_H, int Nq, int Nk, long long ldm,
                       unsigned char *flags, size_t flags_bytes, void *stream) {
    if (mask_B < 1 || mask_H < 1 || Nq < 0 || Nk < 0) return FA_ERR_INVALID_ARG;
    if (mask_B > 65535 || mask_H > 65535 || static_cast<long long>(mask_B) * mask_H > 65535)
        return FA_ERR_INVALID_ARG;   // one grid slice per plane
    const size_t need = fa_mask_tile_flags_bytes(mask_B, mask_H, Nq, Nk);
    if (need == 0) return FA_OK;
    int st = check_mask(mask, mask_B, mask_H, Nq, Nk, mask_B, mask_H, ldm);
    if (st != FA_OK) return st;
    if (!flags || flags_bytes < need) return FA_ERR_INVALID_ARG;
    int dev;
    if ((st = current_device(&dev)) != FA_OK) return st;
    int *err = nullptr;
    if ((st = device_setup(dev, &err)) != FA_OK) return st;
    cudaError_t e = fa::launch_mask_tile_flags(mask, mask_B * mask_H, Nq, Nk, ldm, flags,
                                               static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_fwd_mask(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H,
                int Nq, int Nk, int D, int causal, float scale, int dtype, const float *mask,
                int mask_B, int mask_H, long long ldm, const unsigned char *tile_flags, void *stream) {
    int st = check_common(B, H, Nq, Nk, D, causal, scale, dtype);
    if (st != FA_OK) return st;
    if (Nq == 0) return FA_OK;
    if ((st = check_mask(mask, B, H, Nq, Nk, mask_B, mask_H, ldm)) != FA_OK) return st;
    if (!q || !o || !lse || (Nk > 0 && (!k || !v))) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_INVALID_ARG;
    int dev;
    if ((st = current_device(&dev)) != FA_OK) return st;
    int *err = nullptr, sms = 1;
    if ((st = device_setup(dev, &err, &sms)) != FA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == FA_BF16;
    const long long BH = static_cast<long long>(B) * H;
    if (Nk == 0) {
        return fa::launch_fwd_empty(o, lse, static_cast<size_t>(BH) * Nq, D, bf16, s) == cudaSuccess
                   ? FA_OK : FA_ERR_CUDA;
    }
    fa::FwdTensorMaps tm;
    if ((st = make_map(&tm.q, q, bf16, D, Nq, BH, 128)) != FA_OK) return st;
    if ((st = make_map(&tm.k, k, bf16, D, Nk, BH, 128)) != FA_OK) return st;
    if ((st = make_map(&tm.v, v, bf16, D, Nk, BH, 128)) != FA_OK) return st;
    fa::FwdParams p = fwd_params(B, H, Nq, Nk, scale, nullptr, o, lse, err);
    p.mask = mask;
    p.mask_B = mask_B;
    p.mask_H = mask_H;
    p.ldm = ldm;
    p.tile_flags = tile_flags;
    cudaError_t e = fa::launch_fwd_mask(tm, p, D, bf16, causal != 0, persistent_grid(p.n_units, sms), s);
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"

namespace {
// Argument checks of the packed variable-length entry points.
int check_varlen(const int *cu_q, const int *cu_k, int num_seqs, int H, int total_q, int total_k,
                 int max_q, int max_k, int D, int causal, float scale, int dtype) {
    int st = check_common(num_seqs, H, max_q, max_k, D, causal, scale, dtype);
    if (st != FA_OK) return st;
    if (!cu_q || !cu_k || (reinterpret_cast<uintptr_t>(cu_q) & 3) || (reinterpret_cast<uintptr_t>(cu_k) & 3))
        return FA_ERR_INVALID_ARG;
    if (total_q < 0 || total_k < 0 || total_q > (1 << 30) || total_k > (1 << 30)) return FA_ERR_INVALID_ARG;
    if (static_cast<long long>(H) * total_q > INT32_MAX || static_cast<long long>(H) * total_k > INT32_MAX)
        return FA_ERR_INVALID_ARG;
    return FA_OK;
}
}  // namespace

extern "C" {

int fa_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                  const int *cu_seqlens_q, const int *cu_seqlens_k, int num_seqs, int H, int total_q,
                  int total_k, int max_seqlen_q, int max_seqlen_k, int D, int causal, float scale,
                  int dtype, void *stream) {
    int st = check_varlen(cu_seqlens_q, cu_seqlens_k, num_seqs, H, total_q, total_k, max_seqlen_q,
                          max_seqlen_k, D, causal, scale, dtype);
    if (st != FA_OK) return st;
    if (total_q == 0 || max_seqlen_q == 0) return FA_OK;
    if (!q || !o || !lse || (total_k > 0 && (!k || !v))) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_INVALID_ARG;
    int dev;
    if ((st = current_device(&dev)) != FA_OK) return st;
    int *err = nullptr, sms = 1;
    if ((st = device_setup(dev, &err, &sms)) != FA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == FA_BF16;
    if (total_k == 0 || max_seqlen_k == 0) {
        return fa::launch_fwd_empty(o, lse, static_cast<size_t>(H) * total_q, D, bf16, s) == cudaSuccess
                   ? FA_OK : FA_ERR_CUDA;
    }
    fa::FwdTensorMaps tm;
    if ((st = make_map(&tm.q, q, bf16, D, total_q, H, 128)) != FA_OK) return st;
    if ((st = make_map(&tm.k, k, bf16, D, total_k, H, 128)) != FA_OK) return st;
    if ((st = make_map(&tm.v, v, bf16, D, total_k, H, 128)) != FA_OK) return st;
    fa::FwdParams p = fwd_params(num_seqs, H, max_seqlen_q, max_seqlen_k, scale, nullptr, o, lse, err);
    p.cu_q = cu_seqlens_q;
    p.cu_k = cu_seqlens_k;
    p.total_q = total_q;
    p.total_k = total_k;
    cudaError_t e = fa::launch_fwd_varlen(tm, p, D, bf16, causal != 0, persistent_grid(p.n_units, sms), s);
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int Nq, int Nk, int D, int num_splits) {
    (void)Nk;
    if (B < 1 || H < 1 || Nq < 0 || (D != 64 && D != 128) || num_splits < 1 || num_splits > 256) return 0;
    const size_t rows = static_cast<size_t>(B) * H * Nq * num_splits;
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    return up(rows * D * sizeof(float)) + up(rows * sizeof(float)) + 256;
}

int fa_fwd_splitkv(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H,
                   int Nq, int Nk, int D, int causal, float scale, int dtype, const float *key_bias,
                   int num_splits, void *workspace, size_t workspace_bytes, void *stream) {
    int st = check_common(B, H, Nq, Nk, D, causal, scale, dtype);
    if (st != FA_OK) return st;
    if (num_splits < 1 || num_splits > 256) return FA_ERR_INVALID_ARG;
    if (Nq == 0) return FA_OK;
    if (num_splits == 1 || Nk == 0)
        return fa_fwd(q, k, v, o, lse, B, H, Nq, Nk, D, causal, scale, dtype, key_bias, stream);
    if (!q || !o || !lse || !k || !v) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
        (key_bias && !aligned16(key_bias)) || !aligned16(workspace))
        return FA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, D, num_splits))
        return FA_ERR_WORKSPACE;
    const long long units = static_cast<long long>(B) * H * ((Nq + 255) / 256) * num_splits;
    if (units > INT32_MAX) return FA_ERR_INVALID_ARG;
    int dev;
    if ((st = current_device(&dev)) != FA_OK) return st;
    int *err = nullptr, sms = 1;
    if ((st = device_setup(dev, &err, &sms)) != FA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == FA_BF16;
    const long long BH = static_cast<long long>(B) * H;
    fa::FwdTensorMaps tm;
    if ((st = make_map(&tm.q, q, bf16, D, Nq, BH, 128)) != FA_OK) return st;
    if ((st = make_map(&tm.k, k, bf16, D, Nk, BH, 128)) != FA_OK) return st;
    if ((st = make_map(&tm.v, v, bf16, D, Nk, BH, 128)) != FA_OK) return st;
    const size_t rows = static_cast<size_t>(BH) * Nq * num_splits;
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    fa::FwdParams p = fwd_params(B, H, Nq, Nk, scale, key_bias, o, lse, err);
    const int tiles = (Nk + 127) / 128;
    p.num_splits = num_splits;
    p.tiles_per_split = (tiles + num_splits - 1) / num_splits;
    p.n_units = static_cast<int>(units);
    p.o_part = static_cast<float *>(workspace);
    p.lse_part = reinterpret_cast<float *>(static_cast<char *>(workspace) + up(rows * D * sizeof(float)));
    cudaError_t e = fa::launch_fwd_split(tm, p, D, bf16, causal != 0, key_bias != nullptr,
                                         persistent_grid(units, sms), s);
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_splitkv_num_splits(int B, int H, int Nq, int Nk, int num_sms) {
    if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || num_sms < 0) return 1;
    if (num_sms == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || num_sms < 1) {
            cudaGetLastError();
            return 1;
        }
    }
    const long long units = static_cast<long long>(B) * H * ((Nq + 255) / 256);
    const int tiles = (Nk + 127) / 128;
    if (units >= num_sms || tiles < 2) return 1;
    long long best_cost = -1;
    int best = 1;
    for (int s = 1; s <= std::min(tiles, 256); ++s) {
        const int per = (tiles + s - 1) / s;          // key tiles per split
        const int used = (tiles + per - 1) / per;     // splits that hold tiles
        if (used != s) continue;                      // the same cut as a smaller count
        const long long waves = (units * s + num_sms - 1) / num_sms;
        const long long cost = waves * (per + 1);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    return best;
}

size_t fa_bwd_workspace_bytes(int B, int H, int Nq, int Nk, int D) {
    (void)Nk;
    if (B < 1 || H < 1 || Nq < 0 || (D != 64 && D != 128)) return 0;
    const size_t rows = static_cast<size_t>(B) * H * Nq;
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    return up(rows * sizeof(float)) + 256;
}

}  // extern "C"

namespace {
// Shared body of fa_bwd and fa_bwd_mask (mask == nullptr: no general mask).
// Packed variable-length sequences of the backward (cu_q == nullptr: fixed layout).
struct VarlenArgs {
    const int *cu_q = nullptr, *cu_k = nullptr;
    int total_q = 0, total_k = 0;
};

int bwd_impl(const void *q, const void *k, const void *v, const void *o, const float *lse,
             const void *dO, void *dq, void *dk, void *dv, int B, int H, int Nq, int Nk, int D,
             int causal, float scale, int dtype, const float *key_bias, const float *mask,
             int mask_B, int mask_H, long long ldm, void *workspace, size_t workspace_bytes,
             void *stream, const VarlenArgs &vl = VarlenArgs{}, const unsigned char *tile_flags = nullptr) {
    const bool varlen = vl.cu_q != nullptr;
    int st = varlen ? check_varlen(vl.cu_q, vl.cu_k, B, H, vl.total_q, vl.total_k, Nq, Nk, D, causal, scale, dtype)
                    : check_common(B, H, Nq, Nk, D, causal, scale, dtype);
    if (st != FA_OK) return st;
    // rows of the q-side and k-side tensors: [B*H, N] or, packed, [H, total]
    const long long q_rows = varlen ? static_cast<long long>(H) * vl.total_q : static_cast<long long>(B) * H * Nq;
    const long long k_rows = varlen ? static_cast<long long>(H) * vl.total_k : static_cast<long long>(B) * H * Nk;
    if (varlen && (vl.total_q == 0 || Nq == 0)) Nq = 0;
    if (varlen && (vl.total_k == 0 || Nk == 0)) Nk = 0;
    if (mask && Nq > 0 && (st = check_mask(mask, B, H, Nq, Nk, mask_B, mask_H, ldm)) != FA_OK) return st;
    if (Nq > 0 && (!q || !o || !lse || !dO || !dq)) return FA_ERR_INVALID_ARG;
    if (Nk > 0 && (!k || !v || !dk || !dv)) return FA_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, o, lse, dO, dq, dk, dv, key_bias, workspace};
    for (const void *ptr : ptrs)
        if (!aligned16(ptr)) return FA_ERR_INVALID_ARG;
    const size_t need = varlen ? fa_bwd_workspace_bytes(1, H, vl.total_q, vl.total_k, D)
                               : fa_bwd_workspace_bytes(B, H, Nq, Nk, D);
    if (Nq > 0 && (!workspace || workspace_bytes < need)) return FA_ERR_WORKSPACE;
    int dev;
    if ((st = current_device(&dev)) != FA_OK) return st;
    int *err = nullptr;
    if ((st = device_setup(dev, &err)) != FA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == FA_BF16;
    const long long BH = static_cast<long long>(B) * H;
    if (Nq == 0) {
        // no query: every key and value gradient is zero
        if (Nk == 0 || k_rows == 0) return FA_OK;
        const size_t bytes = static_cast<size_t>(k_rows) * D * 2;
        if (cudaMemsetAsync(dk, 0, bytes, s) != cudaSuccess || cudaMemsetAsync(dv, 0, bytes, s) != cudaSuccess)
            return FA_ERR_CUDA;
        return FA_OK;
    }
    if (Nk == 0) {
        // no key: every output row is empty, so dQ is zero
        if (cudaMemsetAsync(dq, 0, static_cast<size_t>(q_rows) * D * 2, s) != cudaSuccess) return FA_ERR_CUDA;
        return FA_OK;
    }
    fa::BwdParams p{};
    p.B = B;
    p.H = H;
    p.Nq = Nq;
    p.Nk = Nk;
    p.causal_off = Nk - Nq;
    p.qk_scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634074);
    p.scale = scale;
    p.bias = key_bias;
    p.mask = mask;
    p.mask_B = mask_B;
    p.mask_H = mask_H;
    p.ldm = ldm;
    p.tile_flags = mask ? tile_flags : nullptr;
    p.lse = lse;
    p.o = o;
    p.dO = dO;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.Di = static_cast<float *>(workspace);
    p.err = err;
    p.timeout_ns = kDefaultTimeoutNs;
    p.cu_q = vl.cu_q;
    p.cu_k = vl.cu_k;
    p.total_q = vl.total_q;
    p.total_k = vl.total_k;
    // tensor maps over [B*H, N, D] or, packed, [H, total, D]
    const int nq_map = varlen ? vl.total_q : Nq, nk_map = varlen ? vl.total_k : Nk;
    const long long z_map = varlen ? H : BH;
    fa::BwdTensorMaps tm;
    {
        if ((st = make_map(&tm.q, q, bf16, D, nq_map, z_map, 128)) != FA_OK) return st;
        if ((st = make_map(&tm.dO, dO, bf16, D, nq_map, z_map, 128)) != FA_OK) return st;
        if ((st = make_map(&tm.k, k, bf16, D, nk_map, z_map, 128)) != FA_OK) return st;
        if ((st = make_map(&tm.v, v, bf16, D, nk_map, z_map, 128)) != FA_OK) return st;
        if ((st = make_map(&tm.dk, dk, bf16, D, nk_map, z_map, 32)) != FA_OK) return st;
        if ((st = make_map(&tm.dv, dv, bf16, D, nk_map, z_map, 32)) != FA_OK) return st;
        if ((st = make_map(&tm.dq, dq, bf16, D, nq_map, z_map, 32)) != FA_OK) return st;
    }
    cudaError_t e = varlen ? fa::launch_bwd_varlen(tm, p, D, bf16, causal != 0, s)
                  : mask ? fa::launch_bwd_mask(tm, p, D, bf16, causal != 0, s)
                         : fa::launch_bwd(tm, p, D, bf16, causal != 0, key_bias != nullptr, s);
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}
}  // namespace

extern "C" {

int fa_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
           const void *dO, void *dq, void *dk, void *dv, int B, int H, int Nq, int Nk, int D,
           int causal, float scale, int dtype, const float *key_bias, void *workspace,
           size_t workspace_bytes, void *stream) {
    return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, B, H, Nq, Nk, D, causal, scale, dtype, key_bias,
                    nullptr, 0, 0, 0, workspace, workspace_bytes, stream);
}

int fa_bwd_varlen(const void *q, const void *k, const void *v, const void *o, const float *lse,
                  const void *dO, void *dq, void *dk, void *dv, const int *cu_seqlens_q,
                  const int *cu_seqlens_k, int num_seqs, int H, int total_q, int total_k,
                  int max_seqlen_q, int max_seqlen_k, int D, int causal, float scale, int dtype,
                  void *workspace, size_t workspace_bytes, void *stream) {
    if (!cu_seqlens_q || !cu_seqlens_k) return FA_ERR_INVALID_ARG;
    VarlenArgs vl;
    vl.cu_q = cu_seqlens_q;
    vl.cu_k = cu_seqlens_k;
    vl.total_q = total_q;
    vl.total_k = total_k;
    return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, num_seqs, H, max_seqlen_q, max_seqlen_k, D, causal,
                    scale, dtype, nullptr, nullptr, 0, 0, 0, workspace, workspace_bytes, stream, vl);
}

int fa_bwd_mask(const void *q, const void *k, const void *v, const void *o, const float *lse,
                const void *dO, void *dq, void *dk, void *dv, int B, int H, int Nq, int Nk, int D,
                int causal, float scale, int dtype, const float *mask, int mask_B, int mask_H,
                long long ldm, const unsigned char *tile_flags, void *workspace, size_t workspace_bytes,
                void *stream) {
    if (!mask) return FA_ERR_INVALID_ARG;
    return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, B, H, Nq, Nk, D, causal, scale, dtype, nullptr,
                    mask, mask_B, mask_H, ldm, workspace, workspace_bytes, stream, VarlenArgs{}, tile_flags);
}

int fa_device_status(void *stream) {
    int dev;
    int st = current_device(&dev);
    if (st != FA_OK) return st;
    int *err = nullptr;
    if ((st = device_setup(dev, &err)) != FA_OK) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
    int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_fa_error_word, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_fa_error_word, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
    return word;
}

}  // extern "C"

// ---- bounded-wait self-test: one warp waits on a barrier nothing completes.
namespace {
__global__ void fa_wait_timeout_kernel(int *err, unsigned long long timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        fa::mbar_init(fa::smem_u32(&bar), 1);
        fa::fence_mbar_init();
    }
    __syncthreads();
    fa::WaitCtx w{timeout_ns, err, &abort_flag};
    fa::mbar_wait(fa::smem_u32(&bar), 0, w);   // no arrive ever comes
    __syncthreads();
    if (threadIdx.x == 0) fa::mbar_arrive(fa::smem_u32(&bar));   // leave the barrier complete
}
}  // namespace

extern "C" int fa_debug_wait_timeout(unsigned timeout_us, void *stream) {
    int dev;
    int st = current_device(&dev);
    if (st != FA_OK) return st;
    int *err = nullptr;
    if ((st = device_setup(dev, &err)) != FA_OK) return st;
    if (timeout_us == 0 || timeout_us > 10000000u) return FA_ERR_INVALID_ARG;
    fa::prof_begin(static_cast<cudaStream_t>(stream), "fa_wait_timeout_kernel");
    fa_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        err, static_cast<unsigned long long>(timeout_us) * 1000ull);
    fa::prof_end(static_cast<cudaStream_t>(stream));
    fa::note_launch();
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// ---- allocation-free backward ----------------------------------------------
// Some callers may not allocate device memory at all once they are running:
// services that reserve their whole memory budget at start-up and forbid
// allocation on the request path, plugin hosts that hand a library only its
// input and output buffers, and latency-critical paths where an allocation's
// cost or possible failure is not acceptable.  fa_bwd_noalloc serves them with
// a fixed scratch array compiled into the library instead of a workspace
// argument.  The array is file-scope device memory: every GPU that loads the
// library holds it until the process exits.
namespace {
constexpr size_t kNoAllocMaxRows = FA_BWD_NOALLOC_MAX_ROWS;
// D_i of every query row (4 bytes per row) plus the 256 bytes of alignment
// slack that fa_bwd_workspace_bytes() counts.
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocMaxRows + 64];
std::mutex g_noalloc_mu;
float *g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// the array's name only stands in for the symbol; the address a kernel may
// use has to be asked of the runtime, once per device.
int noalloc_scratch(int dev, float **out) {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
            return FA_ERR_CUDA;
        g_noalloc_addr[dev] = static_cast<float *>(ptr);
    }
    *out = g_noalloc_addr[dev];
    return FA_OK;
}
}  // namespace

extern "C" int fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                              const float *lse, const void *dO, void *dq, void *dk, void *dv, int B,
                              int H, int Nq, int Nk, int D, int causal, float scale, int dtype,
                              const float *key_bias, void *stream) {
    // Argument errors first, with the same codes as fa_bwd(); then the size
    // limit of the fixed scratch; both before any CUDA call.
    int st = check_common(B, H, Nq, Nk, D, causal, scale, dtype);
    if (st != FA_OK) return st;
    if (static_cast<long long>(B) * H * Nq > static_cast<long long>(kNoAllocMaxRows))
        return FA_ERR_WORKSPACE;
    // The device must be usable (an sm_100 GPU) before the scratch array's
    // address is asked for: on any other device the library has no image and
    // the lookup would fail with a less precise code.
    int dev;
    if ((st = current_device(&dev)) != FA_OK) return st;
    int *err = nullptr;
    if ((st = device_setup(dev, &err)) != FA_OK) return st;
    float *scratch = nullptr;
    if ((st = noalloc_scratch(dev, &scratch)) != FA_OK) return st;
    // Every scratch entry the kernels read is written earlier in the same call
    // (the row-term pre-pass covers every query row), so nothing needs clearing.
    return fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, Nq, Nk, D, causal, scale, dtype, key_bias,
                  scratch, sizeof(g_noalloc_scratch), stream);
}
