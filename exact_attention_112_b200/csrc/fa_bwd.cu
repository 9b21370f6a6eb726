// fa_bwd.cu -- exact-attention backward for sm_100a (B200).
//
// The backward pass recomputes the scores from Q, K and the saved row
// log-sum-exp instead of storing S or P (lastdictionary.com, "FlashAttention",
// definition paragraph; the two-pass backward of the algebra digest
// "Mastering FlashAttention").  The gradient formulas are not printed on the
// pages; they follow from differentiating O = softmax(scale QK^T + mask) V
// with L = sum(O * dO):
//
//   P  = exp(scale Q K^T + mask - LSE)        (recomputed, never stored)
//   dV = P^T dO        dP = dO V^T
//   dS = P * (dP - D)  with D_i = sum_j P_ij dP_ij = rowsum(dO * O)
//   dQ = scale dS K    dK = scale dS^T Q
//
// Three kernels on one stream:
//   1. fa_bwd_pre_kernel     D_i = rowsum(dO * O) (fp32) and dQacc = 0.
//   2. fa_bwd_dkdv_kernel    one CTA per (b, h, 128-key tile).  For every
//      query tile j that can see these keys:
//        S^T  = K Q_j^T, dP^T = V dO_j^T          tcgen05.mma -> tensor memory
//        P^T  = 2^(S^T qk_scale + bias - LSE_2)    one thread per key row
//        dS^T = P^T * (dP^T - D_j)
//        dV  += P^T dO_j   (P^T from tensor memory)
//        dK  += dS^T Q_j   (dS^T from shared memory, K-major)
//        dQ_j = dS K       (the same dS^T buffer read as an MN-major operand)
//      and a readout warpgroup adds scale * dQ_j into dQacc with TMA bulk
//      reduce-add (fp32).  dK (x scale) and dV are written once at the end.
//   3. fa_bwd_dq_convert_kernel  dQ = dQacc cast to the 16-bit type.
//
// Tensor memory of the dK/dV kernel (lane = key row, except dQ: lane = query):
//   cols [0,128)      S^T (fp32); P^T (16-bit pairs) overwrites cols [0,64)
//   cols [128,256)    dP^T (fp32); dQ_j (fp32) in cols [128,128+D) once dS^T
//                     has been formed from it
//   cols [256,256+D)  dV accumulator,  cols [256+D,256+2D) dK accumulator
// Warp roles (10 warps): 0-3 recompute/gradient, 4-7 dQ readout, 8 TMA
// producer (also stages LSE and D of each query tile), 9 MMA issuer.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

constexpr int kBK = 128;          // keys per CTA tile (MMA M for S^T, dP^T, dV, dK)
constexpr int kBQ = 128;          // queries per step
constexpr int kThreads = 320;
constexpr int kReadoutWarp0 = 4;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BwdLayout {
    static constexpr int kTileBytes = 128 * D * 2;
    static constexpr int kChunkBytes = 128 * 128;     // 128 rows x 64 16-bit values
    static constexpr int kK = 0;
    static constexpr int kV = kK + kTileBytes;
    static constexpr int kQ = kV + kTileBytes;        // 2 stages
    static constexpr int kDO = kQ + 2 * kTileBytes;   // 2 stages
    static constexpr int kDS = kDO + 2 * kTileBytes;  // dS^T: 128 keys x 128 queries, 16-bit
    static constexpr int kRow = kDS + 128 * 128 * 2;  // 2 stages x {LSE_2[128], D[128]} f32
    static constexpr int kBar = kRow + 2 * 2 * 128 * 4;
    static constexpr int kKVFull = 0;
    static constexpr int kQFull = 1;    // +stage
    static constexpr int kQEmpty = 3;   // +stage
    static constexpr int kSFull = 5;
    static constexpr int kPTFull = 6;
    static constexpr int kDPFull = 7;
    static constexpr int kDSFull = 8;
    static constexpr int kDQFull = 9;
    static constexpr int kDQEmpty = 10;
    static constexpr int kAccFull = 11;
    static constexpr int kDrain = 12;
    static constexpr int kNumBars = 13;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 128, kColDV = 256, kColDK = 256 + D;
};

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }
__device__ __forceinline__ float pos_inf() { return __int_as_float(0x7f800000); }

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if constexpr (BF16) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&h);
    } else {
        __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&h);
    }
}

template <bool BF16>
__device__ __forceinline__ float2 unpack2(uint32_t u) {
    if constexpr (BF16) {
        __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162 *>(&u);
        return __bfloat1622float2(h);
    } else {
        __half2 h = *reinterpret_cast<__half2 *>(&u);
        return __half22float2(h);
    }
}

// ---------------------------------------------------------------------------
// 1. D_i = rowsum(dO * O) and dQacc = 0.  One warp per row.
// ---------------------------------------------------------------------------
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const uint16_t *__restrict__ o,
                                                         const uint16_t *__restrict__ dO,
                                                         float *__restrict__ Di,
                                                         float *__restrict__ dq_acc,
                                                         long long rows) {
    const long long warp_global = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    for (long long r = warp_global; r < rows; r += nwarps) {
        constexpr int kPer = D / 32;   // 16-bit values per lane (2 or 4)
        const uint16_t *orow = o + r * D + lane * kPer;
        const uint16_t *drow = dO + r * D + lane * kPer;
        float acc = 0.f;
        if constexpr (kPer == 4) {
            const uint2 a = *reinterpret_cast<const uint2 *>(orow);
            const uint2 b = *reinterpret_cast<const uint2 *>(drow);
            const float2 a0 = unpack2<BF16>(a.x), a1 = unpack2<BF16>(a.y);
            const float2 b0 = unpack2<BF16>(b.x), b1 = unpack2<BF16>(b.y);
            acc = a0.x * b0.x + a0.y * b0.y + a1.x * b1.x + a1.y * b1.y;
        } else {
            const uint32_t a = *reinterpret_cast<const uint32_t *>(orow);
            const uint32_t b = *reinterpret_cast<const uint32_t *>(drow);
            const float2 a0 = unpack2<BF16>(a), b0 = unpack2<BF16>(b);
            acc = a0.x * b0.x + a0.y * b0.y;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) Di[r] = acc;
        float4 *z = reinterpret_cast<float4 *>(dq_acc + r * D);
        for (int c = lane; c < D / 4; c += 32) z[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// ---------------------------------------------------------------------------
// 3. dQ = dQacc (already scaled) cast to 16 bits.
// ---------------------------------------------------------------------------
template <bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_dq_convert_kernel(const float4 *__restrict__ acc,
                                                                uint2 *__restrict__ dq,
                                                                long long n4) {
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
        const float4 a = acc[i];
        dq[i] = make_uint2(pack2<BF16>(a.x, a.y), pack2<BF16>(a.z, a.w));
    }
}

// ---------------------------------------------------------------------------
// 2. dK, dV (and dQ contributions) for one 128-key tile per CTA.
//
// MMA issue order per query tile j (one thread, in-order tensor pipe):
//     dV(j)   after P^T(j) is in tensor memory       (softmax phase 1)
//     dK(j)   after dS^T(j) is in shared memory      (softmax phase 2)
//     S^T(j+1)                                       -> softmax phase 1 of j+1
//     dQ(j)   into the dP^T columns
//     dP^T(j+1) after dQ(j) has been read out        -> softmax phase 2 of j+1
// so the exponentials of tile j+1 overlap dQ(j), its readout and dP^T(j+1).
// ---------------------------------------------------------------------------
template <int D, bool BF16, bool CAUSAL, bool HAS_BIAS>
__global__ void __launch_bounds__(kThreads, 1)
fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                   const __grid_constant__ CUtensorMap tm_dqacc, const BwdParams p) {
    using L = BwdLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    // The layout needs 1024-byte alignment for the 128-byte swizzle atoms; the
    // dynamic shared window starts aligned when no static shared memory is used.
    if ((smem_u32(smem_raw) & 1023u) != 0) {
        if (threadIdx.x == 0) atomicCAS(p.err, 0, kErrInternal);
        return;
    }
    uint8_t *smem = smem_raw;
    const uint32_t sbase = smem_u32(smem);
    auto bar = [&](int i) -> uint32_t { return sbase + L::kBar + 8 * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- work unit: the key tiles that see the most query tiles come first
    const int BH = p.B * p.H;
    const int t = blockIdx.x / BH;
    const int bh = blockIdx.x % BH;
    const int kv0 = t * kBK;
    const int n_q_all = (p.Nq + kBQ - 1) / kBQ;
    int j_begin = 0;
    if (CAUSAL) {
        const int first_q = kv0 - p.causal_off;      // first query that sees key kv0
        j_begin = first_q > 0 ? first_q / kBQ : 0;
        if (j_begin > n_q_all) j_begin = n_q_all;
    }
    const int nq = n_q_all - j_begin;

    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(bar(L::kKVFull), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(L::kQFull + s), 2);   // TMA bytes + the producer's row-term stores
            mbar_init(bar(L::kQEmpty + s), 1);
        }
        mbar_init(bar(L::kSFull), 1);
        mbar_init(bar(L::kPTFull), 128);
        mbar_init(bar(L::kDPFull), 1);
        mbar_init(bar(L::kDSFull), 128);
        mbar_init(bar(L::kDQFull), 1);
        mbar_init(bar(L::kDQEmpty), 128);
        mbar_init(bar(L::kAccFull), 1);
        mbar_init(bar(L::kDrain), 1);
        fence_mbar_init();
    }
    if (warp == kProducerWarp && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_do);
        prefetch_tmap(&tm_dk);
        prefetch_tmap(&tm_dv);
        prefetch_tmap(&tm_dqacc);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtx wctx{p.timeout_ns, p.err, abort_flag};
    const float *lse_bh = p.lse + static_cast<size_t>(bh) * p.Nq;
    const float *di_bh = p.Di + static_cast<size_t>(bh) * p.Nq;

    if (warp == kProducerWarp) {
        // ===================== producer =====================
        bool ok = true;
        int issued = 0;
        if (lane == 0) {
            mbar_arrive_expect_tx(bar(L::kKVFull), 2 * L::kTileBytes);
            for (int c = 0; c < D / 64; ++c) {
                tma_load_3d(sbase + L::kK + c * L::kChunkBytes, &tm_k, bar(L::kKVFull), c * 64, kv0, bh);
                tma_load_3d(sbase + L::kV + c * L::kChunkBytes, &tm_v, bar(L::kKVFull), c * 64, kv0, bh);
            }
        }
        for (int jj = 0; jj < nq; ++jj) {
            const int s = jj & 1;
            const uint32_t ph = (jj >> 1) & 1;
            const int q0 = (j_begin + jj) * kBQ;
            const bool got = mbar_wait(bar(L::kQEmpty + s), ph ^ 1, wctx);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(L::kQFull + s), 2 * L::kTileBytes);
                for (int c = 0; c < D / 64; ++c) {
                    tma_load_3d(sbase + L::kQ + s * L::kTileBytes + c * L::kChunkBytes, &tm_q,
                                bar(L::kQFull + s), c * 64, q0, bh);
                    tma_load_3d(sbase + L::kDO + s * L::kTileBytes + c * L::kChunkBytes, &tm_do,
                                bar(L::kQFull + s), c * 64, q0, bh);
                }
            }
            // row terms of this query tile: LSE in log2 units (+inf for rows
            // that must contribute nothing: past Nq or with no visible key)
            // and D_i.
            float *rowbuf = reinterpret_cast<float *>(smem + L::kRow) + s * 256;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = lane * 4 + e;
                const int q = q0 + r;
                float l2 = pos_inf(), dd = 0.f;
                if (q < p.Nq) {
                    const float l = __ldg(lse_bh + q);
                    l2 = (l == neg_inf()) ? pos_inf() : l * kLog2e;
                    dd = __ldg(di_bh + q);
                }
                rowbuf[r] = l2;
                rowbuf[128 + r] = dd;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::kQFull + s));
            issued = jj + 1;
        }
        if (!ok && lane == 0) {
            WaitCtx drain{wctx.timeout_ns, wctx.err, nullptr};
            volatile int zero = 0;
            drain.abort_flag = &zero;
            mbar_wait(bar(L::kKVFull), 0, drain);
            for (int jj = (issued > 2 ? issued - 2 : 0); jj < issued; ++jj)
                mbar_wait(bar(L::kQFull + (jj & 1)), (jj >> 1) & 1, drain);
        }
    } else if (warp == kMmaWarp) {
        // ===================== MMA issuer =====================
        if (lane == 0) {
            constexpr uint32_t idesc_st = idesc_f16_f32acc(BF16, kBK, kBQ, false, false);  // S^T, dP^T
            constexpr uint32_t idesc_dv = idesc_f16_f32acc(BF16, kBK, D, false, true);     // dV, dK
            constexpr uint32_t idesc_dq = idesc_f16_f32acc(BF16, kBQ, D, true, true);      // dQ
            const uint32_t sK = sbase + L::kK, sV = sbase + L::kV, sDS = sbase + L::kDS;
            auto issue_st = [&](int s) {   // S^T = K Q^T (both K-major)
                const uint32_t sQ = sbase + L::kQ + s * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * L::kChunkBytes + (kk & 3) * 32;
                    umma_f16_ss(tmem + L::kColS, smem_desc_sw128(sK + off, 16, 1024),
                                smem_desc_sw128(sQ + off, 16, 1024), idesc_st, kk > 0);
                }
            };
            auto issue_dpt = [&](int s) {  // dP^T = V dO^T (both K-major)
                const uint32_t sDO = sbase + L::kDO + s * L::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * L::kChunkBytes + (kk & 3) * 32;
                    umma_f16_ss(tmem + L::kColDP, smem_desc_sw128(sV + off, 16, 1024),
                                smem_desc_sw128(sDO + off, 16, 1024), idesc_st, kk > 0);
                }
            };
            bool ok = mbar_wait(bar(L::kKVFull), 0, wctx);
            if (ok && nq > 0) {
                ok = mbar_wait(bar(L::kQFull + 0), 0, wctx);
                if (ok) {
                    tc_fence_after();
                    issue_st(0);
                    umma_commit(bar(L::kSFull));
                    issue_dpt(0);
                    umma_commit(bar(L::kDPFull));
                }
            }
            for (int jj = 0; jj < nq && ok; ++jj) {
                const int s = jj & 1;
                const uint32_t sQ = sbase + L::kQ + s * L::kTileBytes;
                const uint32_t sDO = sbase + L::kDO + s * L::kTileBytes;
                const bool more = jj + 1 < nq;
                // dV += P^T dO   (A: P^T in tensor memory; B: dO rows, MN-major)
                if (!mbar_wait(bar(L::kPTFull), jj & 1, wctx)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kBQ / 16; ++kk)
                    umma_f16_ts(tmem + L::kColDV, tmem + L::kColS + kk * 8,
                                smem_desc_sw128(sDO + kk * 2048, L::kChunkBytes, 1024), idesc_dv,
                                (jj > 0 || kk > 0) ? 1u : 0u);
                // dK += dS^T Q   (A: dS^T K-major in shared memory; B: Q rows, MN-major)
                if (!mbar_wait(bar(L::kDSFull), jj & 1, wctx)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kBQ / 16; ++kk)
                    umma_f16_ss(tmem + L::kColDK,
                                smem_desc_sw128(sDS + (kk >> 2) * L::kChunkBytes + (kk & 3) * 32, 16, 1024),
                                smem_desc_sw128(sQ + kk * 2048, L::kChunkBytes, 1024), idesc_dv,
                                (jj > 0 || kk > 0) ? 1u : 0u);
                if (more) {
                    const int s2 = (jj + 1) & 1;
                    if (!mbar_wait(bar(L::kQFull + s2), ((jj + 1) >> 1) & 1, wctx)) { ok = false; break; }
                    tc_fence_after();
                    issue_st(s2);
                    umma_commit(bar(L::kSFull));
                }
                // dQ_j = dS K into the dP^T columns (A: dS^T read MN-major; B: K rows, MN-major)
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk)
                    umma_f16_ss(tmem + L::kColDQ, smem_desc_sw128(sDS + kk * 2048, L::kChunkBytes, 1024),
                                smem_desc_sw128(sK + kk * 2048, L::kChunkBytes, 1024), idesc_dq, kk > 0);
                umma_commit(bar(L::kDQFull));
                if (jj + 2 < nq) umma_commit(bar(L::kQEmpty + s));
                if (more) {
                    if (!mbar_wait(bar(L::kDQEmpty), jj & 1, wctx)) { ok = false; break; }
                    tc_fence_after();
                    issue_dpt((jj + 1) & 1);
                    umma_commit(bar(L::kDPFull));
                }
            }
            umma_commit(bar(L::kAccFull));
            umma_commit(bar(L::kDrain));
            WaitCtx drain{wctx.timeout_ns, wctx.err, nullptr};
            volatile int zero = 0;
            drain.abort_flag = &zero;
            mbar_wait(bar(L::kDrain), 0, drain);
        }
    } else if (warp >= kReadoutWarp0) {
        // ===================== dQ readout: TMEM -> smem -> TMA add =====================
        // Each warp stages its 32 rows x 64 columns (fp32, two 32x32 boxes with
        // the 128-byte swizzle) in its quarter of the dS^T buffer, which no MMA
        // reads between dQ(j) completing and dP^T(j+1) being issued.
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const uint32_t tl = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        uint8_t *stage = smem + L::kDS + wq * 8192;
        const uint32_t stage_a = sbase + L::kDS + wq * 8192;
        for (int jj = 0; jj < nq; ++jj) {
            const bool got = mbar_wait(bar(L::kDQFull), jj & 1, wctx);
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            const int q_row0 = (j_begin + jj) * kBQ + wq * 32;
#pragma unroll
            for (int half = 0; half < D / 64; ++half) {
#pragma unroll
                for (int box = 0; box < 2; ++box) {
                    uint32_t v[32];
                    tmem_ld32dp_x32_wait(tl + L::kColDQ + half * 64 + box * 32, v);
                    uint8_t *rowp = stage + box * 4096 + lane * 128;
#pragma unroll
                    for (int k4 = 0; k4 < 8; ++k4) {
                        const int pos = k4 ^ (lane & 7);
                        *reinterpret_cast<float4 *>(rowp + pos * 16) =
                            make_float4(__uint_as_float(v[4 * k4]) * p.scale, __uint_as_float(v[4 * k4 + 1]) * p.scale,
                                        __uint_as_float(v[4 * k4 + 2]) * p.scale, __uint_as_float(v[4 * k4 + 3]) * p.scale);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && q_row0 < p.Nq) {
                    tma_reduce_add_3d(&tm_dqacc, stage_a, half * 64, q_row0, bh);
                    tma_reduce_add_3d(&tm_dqacc, stage_a + 4096, half * 64 + 32, q_row0, bh);
                    tma_store_commit();
                    tma_store_wait_read_all();
                }
                __syncwarp();
            }
            tc_fence_before();
            mbar_arrive(bar(L::kDQEmpty));
        }
        if (lane == 0) tma_store_wait_all();
        (void)row;
    } else {
        // ===================== recompute P^T, dS^T (one thread per key) =====================
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const int key = kv0 + row;
        const uint32_t tl = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        const float qk = p.qk_scale_log2;
        float b2 = key < p.Nk ? 0.f : neg_inf();
        if (HAS_BIAS && key < p.Nk)
            b2 = __ldg(p.bias + static_cast<size_t>(bh / p.H) * p.Nk + key) * kLog2e;
        uint8_t *ds_row = smem + L::kDS + row * 128;
        bool ok = true;
        for (int jj = 0; jj < nq; ++jj) {
            const int s = jj & 1;
            const int q0 = (j_begin + jj) * kBQ;
            const float *rowbuf = reinterpret_cast<const float *>(smem + L::kRow) + s * 256;
            // ---- phase 1: P^T = 2^(S^T qk + bias - LSE_2), to tensor memory
            {
                const bool got = mbar_wait(bar(L::kSFull), jj & 1, wctx);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            }
            tc_fence_after();
            const bool diag = CAUSAL && (key > q0 + p.causal_off);   // some column masked
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t sv[32];
                tmem_ld32dp_x32_wait(tl + L::kColS + c * 32, sv);
                const float4 *l4 = reinterpret_cast<const float4 *>(rowbuf + c * 32);
                uint32_t pp[16];
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    const float4 lv = l4[e4];
                    const float la[4] = {lv.x, lv.y, lv.z, lv.w};
                    float pe[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int e = 4 * e4 + u;
                        float x = fmaf(__uint_as_float(sv[e]), qk, b2 - la[u]);
                        if (diag && key > q0 + c * 32 + e + p.causal_off) x = neg_inf();
                        pe[u] = ex2_approx(x);
                    }
                    pp[2 * e4] = pack2<BF16>(pe[0], pe[1]);
                    pp[2 * e4 + 1] = pack2<BF16>(pe[2], pe[3]);
                }
                tmem_st32dp_x16(tl + L::kColS + c * 16, pp);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(L::kPTFull));
            // ---- phase 2: dS^T = P^T (dP^T - D), to shared memory
            {
                const bool got = mbar_wait(bar(L::kDPFull), jj & 1, wctx);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            }
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pv[16], dpv[32];
                tmem_ld32dp_x16_wait(tl + L::kColS + c * 16, pv);
                tmem_ld32dp_x32_wait(tl + L::kColDP + c * 32, dpv);
                const float4 *d4 = reinterpret_cast<const float4 *>(rowbuf + 128 + c * 32);
                uint32_t dd[16];
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    const float4 dv = d4[e4];
                    const float2 p01 = unpack2<BF16>(pv[2 * e4]);
                    const float2 p23 = unpack2<BF16>(pv[2 * e4 + 1]);
                    const float ds0 = p01.x * (__uint_as_float(dpv[4 * e4 + 0]) - dv.x);
                    const float ds1 = p01.y * (__uint_as_float(dpv[4 * e4 + 1]) - dv.y);
                    const float ds2 = p23.x * (__uint_as_float(dpv[4 * e4 + 2]) - dv.z);
                    const float ds3 = p23.y * (__uint_as_float(dpv[4 * e4 + 3]) - dv.w);
                    dd[2 * e4] = pack2<BF16>(ds0, ds1);
                    dd[2 * e4 + 1] = pack2<BF16>(ds2, ds3);
                }
                // dS^T row into shared memory, 128-byte swizzled, 64 queries per chunk
                const int chunk = (c * 32) / 64;
                const int k16_base = ((c * 32) % 64) / 8;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int k16 = (k16_base + q4) ^ (row & 7);
                    *reinterpret_cast<uint4 *>(ds_row + chunk * L::kChunkBytes + k16 * 16) =
                        make_uint4(dd[4 * q4], dd[4 * q4 + 1], dd[4 * q4 + 2], dd[4 * q4 + 3]);
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            mbar_arrive(bar(L::kDSFull));
        }

        // ---- epilogue: dV and scale * dK, 16-bit, via the (now idle) K and V buffers
        if (ok) {
            const bool got = mbar_wait(bar(L::kAccFull), 0, wctx);
            ok = __all_sync(0xffffffffu, got);
            tc_fence_after();
        }
        if (ok) {
#pragma unroll
            for (int which = 0; which < 2; ++which) {       // 0: dV, 1: dK
                const uint32_t col = which ? L::kColDK : L::kColDV;
                const float mul = which ? p.scale : 1.f;
                uint8_t *stage = smem + (which ? L::kK : L::kV);
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t v[32];
                    if (nq > 0) {
                        tmem_ld32dp_x32_wait(tl + col + cc * 32, v);
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = 0u;
                    }
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = pack2<BF16>(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
                    const int chunk = (cc * 32) / 64;
                    const int k16_base = ((cc * 32) % 64) / 8;
                    uint8_t *rowp = stage + chunk * L::kChunkBytes + row * 128;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int k16 = (k16_base + q4) ^ (row & 7);
                        *reinterpret_cast<uint4 *>(rowp + k16 * 16) =
                            make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                    }
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            const int row0 = kv0 + wq * 32;
            if (lane == 0 && row0 < p.Nk) {
                for (int c = 0; c < D / 64; ++c) {
                    tma_store_3d(&tm_dv, sbase + L::kV + c * L::kChunkBytes + wq * 32 * 128, c * 64, row0, bh);
                    tma_store_3d(&tm_dk, sbase + L::kK + c * L::kChunkBytes + wq * 32 * 128, c * 64, row0, bh);
                }
                tma_store_commit();
                tma_store_wait_all();
            }
        }
        tc_fence_before();
    }

    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
    }
}

template <int D, bool BF16, bool CAUSAL, bool HAS_BIAS>
cudaError_t launch_dkdv_t(const BwdTensorMaps &tm, const BwdParams &p, cudaStream_t stream) {
    using L = BwdLayout<D>;
    auto kern = fa_bwd_dkdv_kernel<D, BF16, CAUSAL, HAS_BIAS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return e;
    const unsigned grid = static_cast<unsigned>((p.Nk + kBK - 1) / kBK) * p.B * p.H;
    kern<<<grid, kThreads, L::kBytes, stream>>>(tm.q, tm.k, tm.v, tm.dO, tm.dk, tm.dv, tm.dqacc, p);
    note_launch();
    return cudaGetLastError();
}

template <int D, bool BF16>
cudaError_t launch_bwd_d(const BwdTensorMaps &tm, const BwdParams &p, bool causal, bool bias,
                         cudaStream_t s) {
    // 1. pre-pass
    {
        const long long rows = static_cast<long long>(p.B) * p.H * p.Nq;
        const unsigned grid = static_cast<unsigned>(std::min<long long>((rows + 7) / 8, 148LL * 16));
        fa_bwd_pre_kernel<D, BF16><<<grid, 256, 0, s>>>(static_cast<const uint16_t *>(p.o),
                                                         static_cast<const uint16_t *>(p.dO), p.Di,
                                                         p.dq_acc, rows);
        note_launch();
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // 2. dK, dV and dQ accumulation
    if (p.Nk > 0) {
        cudaError_t e;
        if (causal)
            e = bias ? launch_dkdv_t<D, BF16, true, true>(tm, p, s) : launch_dkdv_t<D, BF16, true, false>(tm, p, s);
        else
            e = bias ? launch_dkdv_t<D, BF16, false, true>(tm, p, s) : launch_dkdv_t<D, BF16, false, false>(tm, p, s);
        if (e != cudaSuccess) return e;
    }
    // 3. dQ to 16 bits
    {
        const long long n4 = static_cast<long long>(p.B) * p.H * p.Nq * D / 4;
        const unsigned grid = static_cast<unsigned>(std::min<long long>((n4 + 255) / 256, 148LL * 16));
        fa_bwd_dq_convert_kernel<BF16><<<grid, 256, 0, s>>>(reinterpret_cast<const float4 *>(p.dq_acc),
                                                             static_cast<uint2 *>(p.dq), n4);
        note_launch();
        return cudaGetLastError();
    }
}

}  // namespace

cudaError_t launch_bwd(const BwdTensorMaps &tm, const BwdParams &p, int D, bool bf16, bool causal,
                       bool has_bias, cudaStream_t stream) {
    if (D == 64) return bf16 ? launch_bwd_d<64, true>(tm, p, causal, has_bias, stream)
                             : launch_bwd_d<64, false>(tm, p, causal, has_bias, stream);
    return bf16 ? launch_bwd_d<128, true>(tm, p, causal, has_bias, stream)
                : launch_bwd_d<128, false>(tm, p, causal, has_bias, stream);
}

}  // namespace fa
