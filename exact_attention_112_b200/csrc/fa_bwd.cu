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
// Packed variable-length sequences (VARLEN instances) read each (sequence,
// head)'s rows through seq_rows() and store dQ, dK, dV row by row.
//
// An optional additive term after scaling -- a per-key bias [B, Nk] or a
// general mask [B or 1, H or 1, Nq, Nk] -- enters P exactly as in the forward
// and receives no gradient.
//
// Three kernels on one stream, none of which stores S, P or dS:
//   1. fa_bwd_pre_kernel   D_i = rowsum(dO * O) (fp32, the caller's workspace).
//   2. fa_bwd_dkdv_kernel  one CTA per (b, h, 128-key tile); for every query
//      tile j that can see these keys:
//        S^T  = K Q_j^T, dP^T = V dO_j^T           tcgen05.mma -> tensor memory
//        P^T  = 2^(S^T qk_scale + bias - LSE_2)     one thread per key row
//        dS^T = P^T * (dP^T - D_j)
//        dV  += P^T dO_j,  dK += dS^T Q_j           A operands from tensor memory
//      dK (x scale) and dV are written once at the end.
//   3. fa_bwd_dq_kernel    one CTA per (b, h, 128-query tile); Q and dO are
//      copied once into tensor memory; for every key tile j it can see:
//      S = Q K_j^T, dP = dO V_j^T (A operands from tensor memory), P and dS as
//      above (one thread per query row), dQ += dS K_j; dQ (x scale) written
//      once.
// dQ is therefore computed without atomics and is bitwise deterministic; the
// price is recomputing S and dP in kernel 3 (7 tile products per pair of
// tiles instead of 5).
//
// Tensor memory of the dK/dV kernel (lane = key row):
//   cols [0,128)      S^T (fp32); then P^T (16-bit pairs) in the first 32 of
//                     the 64 columns each recompute warpgroup read
//   cols [128,256)    dP^T (fp32); then dS^T (16-bit pairs) likewise
//   cols [256,256+D)  dV accumulator,  cols [256+D,256+2D) dK accumulator
// Tensor memory of the dQ kernel (lane = query row):
//   cols [0,128)      S (fp32)
//   cols [128,256)    dP (fp32); then dS (16-bit pairs) in the first 32 of
//                     the 64 columns each recompute warpgroup read
//   cols [256,256+D)  dQ accumulator
//   then Q and dO of the CTA's query tile as 16-bit pairs (D/2 columns each),
//   the A operands of S and dP
// Warp roles (12 warps): 0-7 recompute/gradient (one thread per tile row and
// half of the tile's columns: warpgroup g owns columns [64g, 64g+64)), 8 TMA
// producer, 9 MMA issuer, 10-11 idle (they complete the third warpgroup for
// the register split).  Every role ends at CTA barrier 1 in its own branch and
// no warp asks for registers after giving them up, so the split cannot
// deadlock.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <type_traits>

#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

constexpr int kBK = 128;          // keys per tile
constexpr int kBQ = 128;          // queries per tile
constexpr int kThreads = 384;     // three warpgroups
constexpr int kRecompute = 256;   // two warpgroups, each owning 64 of a tile's 128 columns
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
// Register split (launch pool 168 x 384 = 64512): recompute warpgroups 192,
// warpgroup 2 (producer, MMA, two idle warps) 120; per SMSP (192+192+120)*32 = 16128.
constexpr uint32_t kRegsRecompute = 192;
constexpr uint32_t kRegsOther = 120;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kEmuEvery = 4;      // one pair of exponentials in kEmuEvery on the FMA pipe

template <int D>
struct DkdvLayout {
    static constexpr int kTileBytes = 128 * D * 2;
    static constexpr int kChunkBytes = 128 * 128;     // 128 rows x 64 16-bit values
    static constexpr int kK = 0;
    static constexpr int kV = kK + kTileBytes;
    static constexpr int kQ = kV + kTileBytes;        // 2 stages
    static constexpr int kDO = kQ + 2 * kTileBytes;   // 2 stages
    static constexpr int kRow = kDO + 2 * kTileBytes; // 2 stages x {LSE_2[128], D[128]} f32
    static constexpr int kBar = kRow + 2 * 2 * 128 * 4;
    static constexpr int kKVFull = 0;
    static constexpr int kQFull = 1;    // +stage
    static constexpr int kQEmpty = 3;   // +stage
    static constexpr int kSFull = 5;
    static constexpr int kPTFull = 6;
    static constexpr int kDPFull = 7;
    static constexpr int kDSFull = 8;
    static constexpr int kAccFull = 9;
    static constexpr int kDrain = 10;
    static constexpr int kNumBars = 11;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static constexpr uint32_t kTmemCols = 512;
    // Each recompute warpgroup g writes its 16-bit results only into columns
    // it has read itself: P^T pairs over its S^T columns [64g, 64g+32) (phase
    // 1), dS^T pairs over its dP^T columns 128 + [64g, 64g+32) (phase 2).  So
    // S^T(j+1) only has to wait for dV(j), and dP^T(j+1) only for dK(j).
    static constexpr uint32_t kColS = 0, kColDP = 128, kColP = 0, kColDS = 128, kColDV = 256,
                              kColDK = 256 + D;
};

template <int D>
struct DqLayout {
    static constexpr int kTileBytes = 128 * D * 2;
    static constexpr int kChunkBytes = 128 * 128;
    static constexpr int kKStages = 3;
    static constexpr int kVStages = 2;
    static constexpr int kQ = 0;                                 // Q, later the dQ staging
    static constexpr int kDO = kQ + kTileBytes;
    static constexpr int kK = kDO + kTileBytes;                  // kKStages
    static constexpr int kV = kK + kKStages * kTileBytes;        // kVStages
    static constexpr int kBias = kV + kVStages * kTileBytes;     // kKStages x 128 f32
    static constexpr int kBar = kBias + kKStages * 128 * 4;
    static constexpr int kQFull = 0;
    static constexpr int kKFull = 1;     // +stage (3)
    static constexpr int kKEmpty = 4;    // +stage (3)
    static constexpr int kVFull = 7;     // +stage (2)
    static constexpr int kVEmpty = 9;    // +stage (2)
    static constexpr int kSFull = 11;
    static constexpr int kSRead = 12;    // every recompute thread has loaded S(j)
    static constexpr int kDPFull = 13;
    static constexpr int kDSFull = 14;
    static constexpr int kQDReady = 15;  // Q and dO are in tensor memory
    static constexpr int kOFull = 16;
    static constexpr int kDrain = 17;
    static constexpr int kNumBars = 18;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static constexpr uint32_t kTmemCols = 512;
    // S, dP (dS over its first 32 columns of each warpgroup half), dQ
    // accumulator, then Q and dO as 16-bit pairs (the A operands of S and dP)
    static constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256, kColQ = 256 + D,
                              kColDO = 256 + D + D / 2;
};
// The dynamic shared memory of a CTA is at most 227 KB; the kernels check at
// run time that the window starts 1024-byte aligned, so no slack is reserved.
static_assert(DkdvLayout<128>::kBytes <= 232448 && DkdvLayout<64>::kBytes <= 232448, "dK/dV shared memory");
static_assert(DqLayout<128>::kBytes <= 232448 && DqLayout<64>::kBytes <= 232448, "dQ shared memory");

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

// With a general mask and its tile summary, the recompute kernels visit only
// the tiles the summary marks: the first query tile q >= from (of key tile
// kt) and the first key tile k >= from (of query tile qt) that must be visited,
// or `end` if none.  Without one, every tile in the range is visited.
template <bool HAS_MASK>
__device__ __forceinline__ int next_qtile(const BwdParams &p, long long plane, int kt, int from, int end) {
    if constexpr (HAS_MASK) {
        if (p.tile_flags != nullptr) {
            for (int q = from; q < end; ++q)
                if (mask_tile_needed(p.tile_flags, plane, p.Nq, p.Nk, q, kt)) return q;
            return end;
        }
    }
    return from;
}

template <bool HAS_MASK>
__device__ __forceinline__ int next_ktile(const BwdParams &p, long long plane, int qt, int from, int end) {
    if constexpr (HAS_MASK) {
        if (p.tile_flags != nullptr) {
            for (int k = from; k < end; ++k)
                if (mask_tile_needed(p.tile_flags, plane, p.Nq, p.Nk, qt, k)) return k;
            return end;
        }
    }
    return from;
}

// ---------------------------------------------------------------------------
// 1. D_i = rowsum(dO * O).  Each lane reads 16 bytes of a row of O and of dO
// (D/8 lanes per row, 32/(D/8) rows per warp-wide load) and a warp issues
// kPreUnroll such loads before it reduces, so that enough bytes are in flight
// to keep HBM busy; the row sum is a butterfly over the row's lanes.
// ---------------------------------------------------------------------------
constexpr int kPreUnroll = 4;

template <bool BF16>
__device__ __forceinline__ float dot8(const uint4 &a, const uint4 &b) {
    const float2 a0 = unpack2<BF16>(a.x), a1 = unpack2<BF16>(a.y), a2 = unpack2<BF16>(a.z), a3 = unpack2<BF16>(a.w);
    const float2 b0 = unpack2<BF16>(b.x), b1 = unpack2<BF16>(b.y), b2 = unpack2<BF16>(b.z), b3 = unpack2<BF16>(b.w);
    return ((a0.x * b0.x + a0.y * b0.y) + (a1.x * b1.x + a1.y * b1.y)) +
           ((a2.x * b2.x + a2.y * b2.y) + (a3.x * b3.x + a3.y * b3.y));
}

template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const uint16_t *__restrict__ o,
                                                         const uint16_t *__restrict__ dO,
                                                         float *__restrict__ Di,
                                                         long long rows) {
    constexpr int kLanes = D / 8;               // 16-byte chunks per row
    constexpr int kRowsPerLoad = 32 / kLanes;   // rows covered by one warp-wide load
    constexpr int kRowsPerIter = kRowsPerLoad * kPreUnroll;
    const int lane = threadIdx.x & 31;
    const int sub = lane / kLanes;              // the lane's row within a load
    const int chunk = lane % kLanes;            // the lane's 16 bytes within the row
    const long long warp_global = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    for (long long r0 = warp_global * kRowsPerIter; r0 < rows; r0 += nwarps * kRowsPerIter) {
        uint4 a[kPreUnroll], b[kPreUnroll];
#pragma unroll
        for (int u = 0; u < kPreUnroll; ++u) {
            const long long r = r0 + u * kRowsPerLoad + sub;
            if (r < rows) {
                a[u] = __ldg(reinterpret_cast<const uint4 *>(o + r * D) + chunk);
                b[u] = __ldg(reinterpret_cast<const uint4 *>(dO + r * D) + chunk);
            } else {
                a[u] = make_uint4(0u, 0u, 0u, 0u);
                b[u] = a[u];
            }
        }
#pragma unroll
        for (int u = 0; u < kPreUnroll; ++u) {
            float acc = dot8<BF16>(a[u], b[u]);
#pragma unroll
            for (int off = kLanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            const long long r = r0 + u * kRowsPerLoad + sub;
            if (chunk == 0 && r < rows) Di[r] = acc;
        }
    }
}

// ---------------------------------------------------------------------------
// Shared pieces of the two recompute kernels.
// ---------------------------------------------------------------------------
// Write 32 consecutive 16-bit values of one row (16 packed pairs starting at
// column col0) into a 128-byte-swizzled staging tile of 128-byte rows, 64
// values per chunk: 16-byte piece k of row r lands at piece k ^ (r % 8).
__device__ __forceinline__ void stage_row_sw128(uint8_t *tile, int row, int col0, const uint32_t (&pk)[16],
                                                int chunk_bytes) {
    const int chunk = col0 / 64;
    const int k16_base = (col0 % 64) / 8;
    uint8_t *rowp = tile + chunk * chunk_bytes + row * 128;
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
        const int k16 = (k16_base + q4) ^ (row & 7);
        *reinterpret_cast<uint4 *>(rowp + k16 * 16) =
            make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
    }
}

// ---------------------------------------------------------------------------
// 2. dK, dV for one 128-key tile per CTA.
//
// MMA issue order per query tile j (one elected lane, in-order tensor pipe):
//     dV(j)        once phase 1 of j has put P^T over the S^T columns
//     S^T(j+1)
//     dK(j)        once phase 2 of j has put dS^T over the dP^T columns
//     dP^T(j+1)
// so S^T(j+1) runs during phase 2 of j and dP^T(j+1) during phase 1 of j+1.
// ---------------------------------------------------------------------------
template <int D, bool BF16, bool CAUSAL, bool HAS_BIAS, bool HAS_MASK = false, bool VARLEN = false>
__global__ void __launch_bounds__(kThreads, 1)
fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                   const BwdParams p) {
    using L = DkdvLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment is needed by the 128-byte swizzle atoms; the dynamic
    // shared window starts aligned when the kernel has no static shared memory.
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
    int t, bh;   // key tile 0 is seen by the most query tiles
    unit_of(blockIdx.x, BH, (p.Nk + kBK - 1) / kBK, t, bh);
    const int kv0 = t * kBK;
    // rows of this (sequence, head): fixed [B*H, N, D] layout or packed sequences
    const SeqRows sr = VARLEN ? seq_rows(bh, p.H, p.Nq, p.Nk, p.cu_q, p.cu_k, p.total_q, p.total_k)
                              : SeqRows{static_cast<long long>(bh) * p.Nq, static_cast<long long>(bh) * p.Nk, p.Nq, p.Nk};
    const int len_q = sr.len_q, len_k = sr.len_k, coff = len_k - len_q;
    const int q_y0 = VARLEN ? static_cast<int>(sr.q_row0 - static_cast<long long>(bh % p.H) * p.total_q) : 0;
    const int k_y0 = VARLEN ? static_cast<int>(sr.k_row0 - static_cast<long long>(bh % p.H) * p.total_k) : 0;
    const int z = VARLEN ? bh % p.H : bh;           // head slice of the tensor maps
    const int n_q_all = kv0 < len_k ? (len_q + kBQ - 1) / kBQ : 0;   // a tile past the keys: no work
    int j_begin = 0;
    if (CAUSAL) {
        const int first_q = kv0 - coff;              // first query that sees key kv0
        j_begin = first_q > 0 ? first_q / kBQ : 0;
        if (j_begin > n_q_all) j_begin = n_q_all;
    }
    const long long plane = HAS_MASK ? mask_plane(bh, p.H, p.mask_B, p.mask_H) : 0;
    int nq = n_q_all - j_begin;      // query tiles this key tile visits
    if (HAS_MASK && p.tile_flags != nullptr) {
        nq = 0;
        for (int q = next_qtile<HAS_MASK>(p, plane, t, j_begin, n_q_all); q < n_q_all;
             q = next_qtile<HAS_MASK>(p, plane, t, q + 1, n_q_all))
            ++nq;
    }

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
        mbar_init(bar(L::kPTFull), kRecompute);
        mbar_init(bar(L::kDPFull), 1);
        mbar_init(bar(L::kDSFull), kRecompute);
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
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtx wctx{p.timeout_ns, p.err, abort_flag};

    if (warp >= 8) regs_release<kRegsOther>();
    if (warp == kProducerWarp) {
        // ===================== producer =====================
        const float *lse_bh = p.lse + sr.q_row0;
        const float *di_bh = p.Di + sr.q_row0;
        bool ok = true;
        int issued = 0;
        if (lane == 0) {
            mbar_arrive_expect_tx(bar(L::kKVFull), 2 * L::kTileBytes);
            for (int c = 0; c < D / 64; ++c) {
                tma_load_3d(sbase + L::kK + c * L::kChunkBytes, &tm_k, bar(L::kKVFull), c * 64, k_y0 + kv0, z);
                tma_load_3d(sbase + L::kV + c * L::kChunkBytes, &tm_v, bar(L::kKVFull), c * 64, k_y0 + kv0, z);
            }
        }
        int qt = next_qtile<HAS_MASK>(p, plane, t, j_begin, n_q_all);   // query tile of step jj
        for (int jj = 0; jj < nq; ++jj, qt = next_qtile<HAS_MASK>(p, plane, t, qt + 1, n_q_all)) {
            const int s = jj & 1;
            const uint32_t ph = (jj >> 1) & 1;
            const int q0 = qt * kBQ;
            const bool got = mbar_wait(bar(L::kQEmpty + s), ph ^ 1, wctx);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(L::kQFull + s), 2 * L::kTileBytes);
                for (int c = 0; c < D / 64; ++c) {
                    tma_load_3d(sbase + L::kQ + s * L::kTileBytes + c * L::kChunkBytes, &tm_q,
                                bar(L::kQFull + s), c * 64, q_y0 + q0, z);
                    tma_load_3d(sbase + L::kDO + s * L::kTileBytes + c * L::kChunkBytes, &tm_do,
                                bar(L::kQFull + s), c * 64, q_y0 + q0, z);
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
                if (q < len_q) {
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
        named_bar_sync(1, kThreads);
    } else if (warp == kMmaWarp) {
        // ===================== MMA issuer (whole warp; one elected lane issues) =====================
        {
            constexpr uint32_t idesc_st = idesc_f16_f32acc(BF16, kBK, kBQ, false, false);  // S^T, dP^T
            constexpr uint32_t idesc_acc = idesc_f16_f32acc(BF16, kBK, D, false, true);    // dV, dK
            const uint64_t dK0 = smem_desc_sw128(sbase + L::kK, 16, 1024);
            const uint64_t dV0 = smem_desc_sw128(sbase + L::kV, 16, 1024);
            auto issue_st = [&](int s) {    // S^T = K Q^T (both K-major)
                const uint64_t dq = smem_desc_sw128(sbase + L::kQ + s * L::kTileBytes, 16, 1024);
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = ((kk >> 2) * L::kChunkBytes + (kk & 3) * 32) >> 4;
                        umma_f16_ss(tmem + L::kColS, dK0 + off, dq + off, idesc_st, kk > 0);
                    }
                    umma_commit(bar(L::kSFull));
                }
                __syncwarp();
            };
            auto issue_dpt = [&](int s) {   // dP^T = V dO^T (both K-major)
                const uint64_t ddo = smem_desc_sw128(sbase + L::kDO + s * L::kTileBytes, 16, 1024);
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = ((kk >> 2) * L::kChunkBytes + (kk & 3) * 32) >> 4;
                        umma_f16_ss(tmem + L::kColDP, dV0 + off, ddo + off, idesc_st, kk > 0);
                    }
                    umma_commit(bar(L::kDPFull));
                }
                __syncwarp();
            };
            bool ok = mbar_wait_warp(bar(L::kKVFull), 0, wctx);
            if (ok && nq > 0) {
                ok = mbar_wait_warp(bar(L::kQFull + 0), 0, wctx);
                if (ok) {
                    tc_fence_after();
                    issue_st(0);
                    issue_dpt(0);
                }
            }
            for (int jj = 0; jj < nq && ok; ++jj) {
                const int s = jj & 1;
                const int s2 = (jj + 1) & 1;
                // dV += P^T dO   (A: P^T over the S^T columns; B: dO rows, MN-major)
                if (!mbar_wait_warp(bar(L::kPTFull), jj & 1, wctx)) { ok = false; break; }
                tc_fence_after();
                {
                    const uint64_t ddo = smem_desc_sw128(sbase + L::kDO + s * L::kTileBytes, L::kChunkBytes, 1024);
                    if (elect_one()) {
#pragma unroll
                        for (int kk = 0; kk < kBQ / 16; ++kk)
                            umma_f16_ts(tmem + L::kColDV, tmem + L::kColP + (kk >> 2) * 64 + (kk & 3) * 8,
                                        ddo + ((kk * 2048) >> 4), idesc_acc, (jj > 0 || kk > 0) ? 1u : 0u);
                    }
                    __syncwarp();
                }
                // S^T(j+1) over P^T(j) (read by dV(j) just before, in order)
                if (jj + 1 < nq) {
                    if (!mbar_wait_warp(bar(L::kQFull + s2), ((jj + 1) >> 1) & 1, wctx)) { ok = false; break; }
                    tc_fence_after();
                    issue_st(s2);
                }
                // dK += dS^T Q   (A: dS^T over the dP^T columns; B: Q rows, MN-major)
                if (!mbar_wait_warp(bar(L::kDSFull), jj & 1, wctx)) { ok = false; break; }
                tc_fence_after();
                {
                    const uint64_t dq = smem_desc_sw128(sbase + L::kQ + s * L::kTileBytes, L::kChunkBytes, 1024);
                    const bool release = jj + 2 < nq;
                    if (elect_one()) {
#pragma unroll
                        for (int kk = 0; kk < kBQ / 16; ++kk)
                            umma_f16_ts(tmem + L::kColDK, tmem + L::kColDS + (kk >> 2) * 64 + (kk & 3) * 8,
                                        dq + ((kk * 2048) >> 4), idesc_acc, (jj > 0 || kk > 0) ? 1u : 0u);
                        if (release) umma_commit(bar(L::kQEmpty + s));
                    }
                    __syncwarp();
                }
                // dP^T(j+1) over dS^T(j) (read by dK(j) just before, in order)
                if (jj + 1 < nq) issue_dpt(s2);
            }
            if (elect_one()) {
                umma_commit(bar(L::kAccFull));
                umma_commit(bar(L::kDrain));
            }
            __syncwarp();
            WaitCtx drain{wctx.timeout_ns, wctx.err, nullptr};
            volatile int zero = 0;
            drain.abort_flag = &zero;
            mbar_wait(bar(L::kDrain), 0, drain);
        }
        named_bar_sync(1, kThreads);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
    } else if (warp < 8) {
        // ===================== recompute P^T, dS^T (one thread per key, 64 queries) =====================
        regs_alloc<kRegsRecompute>();
        const int g = warp >> 2;            // column half: queries [64g, 64g+64) of each tile
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const int key = kv0 + row;
        const uint32_t tl = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        const float qk = p.qk_scale_log2;
        float b2 = key < len_k ? 0.f : neg_inf();
        if (HAS_BIAS && key < p.Nk)
            b2 = __ldg(p.bias + static_cast<size_t>(bh / p.H) * p.Nk + key) * kLog2e;
        // column `key` of the general mask: M[q][key] for the thread's queries
        // (consecutive keys across the warp, so every load is one 128-byte line)
        const float *mcol = nullptr;
        if (HAS_MASK && key < p.Nk)
            mcol = p.mask + plane * p.Nq * p.ldm + key;
        bool ok = true;
        int qt = next_qtile<HAS_MASK>(p, plane, t, j_begin, n_q_all);   // query tile of step jj
        for (int jj = 0; jj < nq; ++jj, qt = next_qtile<HAS_MASK>(p, plane, t, qt + 1, n_q_all)) {
            const int s = jj & 1;
            const int qg = qt * kBQ + 64 * g;                 // first query of this thread's half
            const float *rowbuf = reinterpret_cast<const float *>(smem + L::kRow) + s * 256 + 64 * g;
            float mk[HAS_MASK ? 64 : 1];
            if constexpr (HAS_MASK) {
                // issued before the wait for S^T so the loads overlap it
#pragma unroll
                for (int e = 0; e < 64; ++e)
                    mk[e] = (mcol != nullptr && qg + e < p.Nq)
                                ? __ldg(mcol + static_cast<long long>(qg + e) * p.ldm) * kLog2e : 0.f;
            }
            // ---- phase 1: P^T = 2^(S^T qk + bias - LSE_2): registers (fp32) and
            // tensor memory (16-bit, the dV operand)
            {
                const bool got = mbar_wait(bar(L::kSFull), jj & 1, wctx);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            }
            tc_fence_after();
            const bool diag = CAUSAL && (key > qg + coff);   // some column masked
            float pr[64];
            {
                uint32_t sv[64];
                tmem_ld32dp_x64_wait(tl + L::kColS + 64 * g, sv);
                const float4 *l4 = reinterpret_cast<const float4 *>(rowbuf);
                const float2 qk2 = make_float2(qk, qk);
                const float2 b22 = make_float2(b2, b2);
                // Without masked scores in this thread's columns, one pair in
                // kEmuEvery takes the FMA-pipe exponential instead of MUFU.
                auto make_p = [&](auto emu_tag) {
                    constexpr bool kEmu = decltype(emu_tag)::value;
#pragma unroll
                    for (int e4 = 0; e4 < 16; ++e4) {
                        const float4 lv = l4[e4];
                        // x = s qk + (bias - LSE_2), two columns per instruction
                        float2 c01 = __fadd2_rn(b22, make_float2(-lv.x, -lv.y));
                        float2 c23 = __fadd2_rn(b22, make_float2(-lv.z, -lv.w));
                        if constexpr (HAS_MASK) {
                            c01 = __fadd2_rn(c01, make_float2(mk[4 * e4], mk[4 * e4 + 1]));
                            c23 = __fadd2_rn(c23, make_float2(mk[4 * e4 + 2], mk[4 * e4 + 3]));
                        }
                        float2 x01 = __ffma2_rn(make_float2(__uint_as_float(sv[4 * e4]), __uint_as_float(sv[4 * e4 + 1])), qk2, c01);
                        float2 x23 = __ffma2_rn(make_float2(__uint_as_float(sv[4 * e4 + 2]), __uint_as_float(sv[4 * e4 + 3])), qk2, c23);
                        if (!kEmu && diag) {
                            const int e = 4 * e4;
                            if (key > qg + e + coff) x01.x = neg_inf();
                            if (key > qg + e + 1 + coff) x01.y = neg_inf();
                            if (key > qg + e + 2 + coff) x23.x = neg_inf();
                            if (key > qg + e + 3 + coff) x23.y = neg_inf();
                        }
                        pr[4 * e4] = ex2_approx(x01.x);
                        pr[4 * e4 + 1] = ex2_approx(x01.y);
                        if (kEmu && (2 * e4 + 1) % kEmuEvery == kEmuEvery - 1) {
                            const float2 p23 = exp2_fma2(x23);
                            pr[4 * e4 + 2] = p23.x;
                            pr[4 * e4 + 3] = p23.y;
                        } else {
                            pr[4 * e4 + 2] = ex2_approx(x23.x);
                            pr[4 * e4 + 3] = ex2_approx(x23.y);
                        }
                    }
                };
                if (__all_sync(0xffffffffu, !HAS_BIAS && !HAS_MASK && !diag && key < len_k))   // warp-uniform
                    make_p(std::true_type{});
                else
                    make_p(std::false_type{});
                // P^T (16-bit) over the first 32 of this thread's S^T columns
                uint32_t pp[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) pp[e] = pack2<BF16>(pr[2 * e], pr[2 * e + 1]);
                tmem_st32dp_x32(tl + L::kColP + 64 * g, pp);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(L::kPTFull));
            // ---- phase 2: dS^T = P^T (dP^T - D), 16-bit, over the dP^T columns
            // this thread has just read
            {
                const bool got = mbar_wait(bar(L::kDPFull), jj & 1, wctx);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            }
            tc_fence_after();
            {
                uint32_t dpv[64];
                tmem_ld32dp_x64_wait(tl + L::kColDP + 64 * g, dpv);
                const float4 *d4 = reinterpret_cast<const float4 *>(rowbuf + 128);
                uint32_t dd[32];
#pragma unroll
                for (int e4 = 0; e4 < 16; ++e4) {
                    const float4 dv = d4[e4];
                    const int e = 4 * e4;
                    const float2 d01 = __fmul2_rn(make_float2(pr[e], pr[e + 1]),
                                                  __fadd2_rn(make_float2(__uint_as_float(dpv[e]), __uint_as_float(dpv[e + 1])),
                                                             make_float2(-dv.x, -dv.y)));
                    const float2 d23 = __fmul2_rn(make_float2(pr[e + 2], pr[e + 3]),
                                                  __fadd2_rn(make_float2(__uint_as_float(dpv[e + 2]), __uint_as_float(dpv[e + 3])),
                                                             make_float2(-dv.z, -dv.w)));
                    dd[2 * e4] = pack2<BF16>(d01.x, d01.y);
                    dd[2 * e4 + 1] = pack2<BF16>(d23.x, d23.y);
                }
                tmem_st32dp_x32(tl + L::kColDS + 64 * g, dd);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(L::kDSFull));
        }

        // ---- epilogue: dV and scale * dK, 16-bit, via the (now idle) K and V buffers
        if (ok) {
            const bool got = mbar_wait(bar(L::kAccFull), 0, wctx);
            ok = __all_sync(0xffffffffu, got);
            tc_fence_after();
        }
        if (ok && VARLEN) {
            // packed sequences: each thread stores its own key row (a 32-row TMA
            // box could run into the next sequence's rows)
            const int which = g;                            // warpgroup 0: dV, 1: dK
            const uint32_t col = which ? L::kColDK : L::kColDV;
            const float mul = which ? p.scale : 1.f;
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(which ? p.dk : p.dv) +
                                                   (sr.k_row0 + key) * D);
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
                if (key < len_k) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        dst[cc * 4 + q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                }
            }
        } else if (ok) {
            {
                const int which = g;                        // warpgroup 0: dV, 1: dK
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
                    stage_row_sw128(stage, row, cc * 32, pk, L::kChunkBytes);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            const int row0 = kv0 + wq * 32;
            if (lane == 0 && row0 < p.Nk) {
                for (int c = 0; c < D / 64; ++c) {
                    if (g == 0)
                        tma_store_3d(&tm_dv, sbase + L::kV + c * L::kChunkBytes + wq * 32 * 128, c * 64, row0, bh);
                    else
                        tma_store_3d(&tm_dk, sbase + L::kK + c * L::kChunkBytes + wq * 32 * 128, c * 64, row0, bh);
                }
                tma_store_commit();
                tma_store_wait_all();
            }
        }
        tc_fence_before();
        named_bar_sync(1, kThreads);
    } else {
        named_bar_sync(1, kThreads);   // idle warps 10, 11
    }
}

// ---------------------------------------------------------------------------
// 3. dQ for one 128-query tile per CTA.
//
// Q and dO are the same for every key tile of the CTA, so the recompute
// warps copy them once into tensor memory and S = Q K_j^T and dP = dO V_j^T
// read their A operand from there: per key tile only K_j and V_j are read
// from shared memory.  MMA issue order per key tile j:
//     S(j+1)     once the recompute warps have loaded S(j) into registers
//     dQ(j)      once dS(j) is over the dP columns
//     dP(j+1)    (over dS(j), read by dQ(j) just before, in order)
// ---------------------------------------------------------------------------
template <int D, bool BF16, bool CAUSAL, bool HAS_BIAS, bool HAS_MASK = false, bool VARLEN = false>
__global__ void __launch_bounds__(kThreads, 1)
fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
    using L = DqLayout<D>;
    extern __shared__ uint8_t smem_raw[];
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

    // ---- work unit: query tiles that see the most key tiles come first
    const int BH = p.B * p.H;
    const int n_q_all = (p.Nq + kBQ - 1) / kBQ;
    int rank_, bh_;
    unit_of(blockIdx.x, BH, n_q_all, rank_, bh_);
    const int qt = (n_q_all - 1) - rank_;
    const int bh = bh_;
    const int q0 = qt * kBQ;
    // rows of this (sequence, head): fixed [B*H, N, D] layout or packed sequences
    const SeqRows sr = VARLEN ? seq_rows(bh, p.H, p.Nq, p.Nk, p.cu_q, p.cu_k, p.total_q, p.total_k)
                              : SeqRows{static_cast<long long>(bh) * p.Nq, static_cast<long long>(bh) * p.Nk, p.Nq, p.Nk};
    const int len_q = sr.len_q, len_k = sr.len_k, coff = len_k - len_q;
    const int q_y0 = VARLEN ? static_cast<int>(sr.q_row0 - static_cast<long long>(bh % p.H) * p.total_q) : 0;
    const int k_y0 = VARLEN ? static_cast<int>(sr.k_row0 - static_cast<long long>(bh % p.H) * p.total_k) : 0;
    const int z = VARLEN ? bh % p.H : bh;           // head slice of the tensor maps
    const int n_kv_all = (len_k + kBK - 1) / kBK;
    int n = q0 < len_q ? n_kv_all : 0;              // a tile past the queries: no work
    if (CAUSAL && n > 0) {
        const int last_row = min(q0 + kBQ - 1, len_q - 1);
        const int lim = last_row + coff;
        n = lim < 0 ? 0 : min(n_kv_all, lim / kBK + 1);
    }
    const int n_range = n;                          // key tiles [0, n_range) may be visible
    const long long plane = HAS_MASK ? mask_plane(bh, p.H, p.mask_B, p.mask_H) : 0;
    if (HAS_MASK && p.tile_flags != nullptr) {     // visit only the tiles the summary marks
        n = 0;
        for (int k = next_ktile<HAS_MASK>(p, plane, qt, 0, n_range); k < n_range;
             k = next_ktile<HAS_MASK>(p, plane, qt, k + 1, n_range))
            ++n;
    }

    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(bar(L::kQFull), 1);
        for (int s = 0; s < L::kKStages; ++s) {
            mbar_init(bar(L::kKFull + s), HAS_BIAS ? 2 : 1);
            mbar_init(bar(L::kKEmpty + s), 1);
        }
        for (int s = 0; s < L::kVStages; ++s) {
            mbar_init(bar(L::kVFull + s), 1);
            mbar_init(bar(L::kVEmpty + s), 1);
        }
        mbar_init(bar(L::kSFull), 1);
        mbar_init(bar(L::kSRead), kRecompute);
        mbar_init(bar(L::kDPFull), 1);
        mbar_init(bar(L::kDSFull), kRecompute);
        mbar_init(bar(L::kQDReady), kRecompute);
        mbar_init(bar(L::kOFull), 1);
        mbar_init(bar(L::kDrain), 1);
        fence_mbar_init();
    }
    if (warp == kProducerWarp && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_do);
        prefetch_tmap(&tm_dq);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtx wctx{p.timeout_ns, p.err, abort_flag};

    if (warp >= 8) regs_release<kRegsOther>();
    if (warp == kProducerWarp) {
        // ===================== producer =====================
        const float *bias_b = HAS_BIAS ? p.bias + static_cast<size_t>(bh / p.H) * p.Nk : nullptr;
        bool ok = true;
        int k_issued = 0, v_issued = 0;
        if (lane == 0 && n > 0) {
            mbar_arrive_expect_tx(bar(L::kQFull), 2 * L::kTileBytes);
            for (int c = 0; c < D / 64; ++c) {
                tma_load_3d(sbase + L::kQ + c * L::kChunkBytes, &tm_q, bar(L::kQFull), c * 64, q_y0 + q0, z);
                tma_load_3d(sbase + L::kDO + c * L::kChunkBytes, &tm_do, bar(L::kQFull), c * 64, q_y0 + q0, z);
            }
        }
        // K runs one tile ahead of V (K_j is needed by S(j), before dP(j)).
        int kt = next_ktile<HAS_MASK>(p, plane, qt, 0, n_range), kt_prev = -1;   // key tiles of steps j, j-1
        for (int j = 0; j < n && ok; ++j, kt_prev = kt, kt = next_ktile<HAS_MASK>(p, plane, qt, kt + 1, n_range)) {
            const int ks = j % L::kKStages;
            const uint32_t kph = (j / L::kKStages) & 1;
            {
                const bool got = mbar_wait(bar(L::kKEmpty + ks), kph ^ 1, wctx);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(L::kKFull + ks), L::kTileBytes);
                for (int c = 0; c < D / 64; ++c)
                    tma_load_3d(sbase + L::kK + ks * L::kTileBytes + c * L::kChunkBytes, &tm_k,
                                bar(L::kKFull + ks), c * 64, k_y0 + kt * kBK, z);
            }
            if constexpr (HAS_BIAS) {
                float *bs = reinterpret_cast<float *>(smem + L::kBias) + ks * 128;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = kt * kBK + lane * 4 + e;
                    bs[lane * 4 + e] = key < p.Nk ? __ldg(bias_b + key) * kLog2e : neg_inf();
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(L::kKFull + ks));
            }
            k_issued = j + 1;
            if (j >= 1) {
                const int jv = j - 1;
                const int vs = jv % L::kVStages;
                const uint32_t vph = (jv / L::kVStages) & 1;
                const bool got = mbar_wait(bar(L::kVEmpty + vs), vph ^ 1, wctx);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(L::kVFull + vs), L::kTileBytes);
                    for (int c = 0; c < D / 64; ++c)
                        tma_load_3d(sbase + L::kV + vs * L::kTileBytes + c * L::kChunkBytes, &tm_v,
                                    bar(L::kVFull + vs), c * 64, k_y0 + kt_prev * kBK, z);
                }
                v_issued = jv + 1;
            }
        }
        if (ok && n > 0) {   // the last V tile
            const int jv = n - 1;
            const int vs = jv % L::kVStages;
            const uint32_t vph = (jv / L::kVStages) & 1;
            const bool got = mbar_wait(bar(L::kVEmpty + vs), vph ^ 1, wctx);
            if (!__all_sync(0xffffffffu, got)) {
                ok = false;
            } else {
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(L::kVFull + vs), L::kTileBytes);
                    for (int c = 0; c < D / 64; ++c)
                        tma_load_3d(sbase + L::kV + vs * L::kTileBytes + c * L::kChunkBytes, &tm_v,
                                    bar(L::kVFull + vs), c * 64, k_y0 + kt_prev * kBK, z);
                }
                v_issued = n;
            }
        }
        if (!ok && lane == 0) {
            WaitCtx drain{wctx.timeout_ns, wctx.err, nullptr};
            volatile int zero = 0;
            drain.abort_flag = &zero;
            if (n > 0) mbar_wait(bar(L::kQFull), 0, drain);
            for (int j = (k_issued > 3 ? k_issued - 3 : 0); j < k_issued; ++j)
                mbar_wait(bar(L::kKFull + j % L::kKStages), (j / L::kKStages) & 1, drain);
            for (int j = (v_issued > 2 ? v_issued - 2 : 0); j < v_issued; ++j)
                mbar_wait(bar(L::kVFull + j % L::kVStages), (j / L::kVStages) & 1, drain);
        }
        named_bar_sync(1, kThreads);
    } else if (warp == kMmaWarp) {
        // ===================== MMA issuer (whole warp; one elected lane issues) =====================
        if (n > 0) {
            constexpr uint32_t idesc_s = idesc_f16_f32acc(BF16, kBQ, kBK, false, false);   // S, dP
            constexpr uint32_t idesc_dq = idesc_f16_f32acc(BF16, kBQ, D, false, true);     // dQ
            auto issue_s = [&](int j) {        // S_j = Q K_j^T   (A: Q in tensor memory)
                const uint64_t dk = smem_desc_sw128(sbase + L::kK + (j % L::kKStages) * L::kTileBytes, 16, 1024);
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        umma_f16_ts(tmem + L::kColS, tmem + L::kColQ + kk * 8,
                                    dk + (((kk >> 2) * L::kChunkBytes + (kk & 3) * 32) >> 4), idesc_s, kk > 0);
                    umma_commit(bar(L::kSFull));
                }
                __syncwarp();
            };
            auto issue_dp = [&](int j) {       // dP_j = dO V_j^T   (A: dO in tensor memory)
                const uint64_t dv = smem_desc_sw128(sbase + L::kV + (j % L::kVStages) * L::kTileBytes, 16, 1024);
                const bool release = j + 2 < n;
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        umma_f16_ts(tmem + L::kColDP, tmem + L::kColDO + kk * 8,
                                    dv + (((kk >> 2) * L::kChunkBytes + (kk & 3) * 32) >> 4), idesc_s, kk > 0);
                    umma_commit(bar(L::kDPFull));
                    if (release) umma_commit(bar(L::kVEmpty + j % L::kVStages));
                }
                __syncwarp();
            };
            bool ok = mbar_wait_warp(bar(L::kQDReady), 0, wctx) && mbar_wait_warp(bar(L::kKFull + 0), 0, wctx);
            if (ok) {
                tc_fence_after();
                issue_s(0);
                ok = mbar_wait_warp(bar(L::kVFull + 0), 0, wctx);
            }
            if (ok) {
                tc_fence_after();
                issue_dp(0);
            }
            for (int j = 0; j < n && ok; ++j) {
                // S(j+1) as soon as every recompute thread holds S(j) in registers
                if (j + 1 < n) {
                    const int js = j + 1;
                    if (!mbar_wait_warp(bar(L::kSRead), j & 1, wctx)) { ok = false; break; }
                    if (!mbar_wait_warp(bar(L::kKFull + js % L::kKStages), (js / L::kKStages) & 1, wctx)) { ok = false; break; }
                    tc_fence_after();
                    issue_s(js);
                }
                // dQ += dS_j K_j  (A: dS over the dP columns; B: K rows, MN-major)
                if (!mbar_wait_warp(bar(L::kDSFull), j & 1, wctx)) { ok = false; break; }
                tc_fence_after();
                {
                    const uint64_t dk = smem_desc_sw128(sbase + L::kK + (j % L::kKStages) * L::kTileBytes,
                                                        L::kChunkBytes, 1024);
                    const bool release = j + 3 < n;
                    if (elect_one()) {
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk)
                            umma_f16_ts(tmem + L::kColDQ, tmem + L::kColDP + (kk >> 2) * 64 + (kk & 3) * 8,
                                        dk + ((kk * 2048) >> 4), idesc_dq, (j > 0 || kk > 0) ? 1u : 0u);
                        if (release) umma_commit(bar(L::kKEmpty + j % L::kKStages));
                    }
                    __syncwarp();
                }
                // dP(j+1) over dS(j)
                if (j + 1 < n) {
                    const int jv = j + 1;
                    if (!mbar_wait_warp(bar(L::kVFull + jv % L::kVStages), (jv / L::kVStages) & 1, wctx)) { ok = false; break; }
                    tc_fence_after();
                    issue_dp(jv);
                }
            }
            if (elect_one()) {
                umma_commit(bar(L::kOFull));
                umma_commit(bar(L::kDrain));
            }
            __syncwarp();
            WaitCtx drain{wctx.timeout_ns, wctx.err, nullptr};
            volatile int zero = 0;
            drain.abort_flag = &zero;
            mbar_wait(bar(L::kDrain), 0, drain);
        }
        named_bar_sync(1, kThreads);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
    } else if (warp < 8) {
        // ===================== recompute P, dS (one thread per query row, 64 keys) =====================
        regs_alloc<kRegsRecompute>();
        const int g = warp >> 2;            // column half: keys [64g, 64g+64) of each tile
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const int q = q0 + row;
        const uint32_t tl = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        const float qk = p.qk_scale_log2;
        bool ok = true;
        if (n > 0) {
            // Q (warpgroup 0) or dO (warpgroup 1) row of this thread: shared
            // memory (128-byte swizzled tile) -> tensor memory, the A operand
            // of S or dP for every key tile of the CTA
            const bool got = mbar_wait(bar(L::kQFull), 0, wctx);
            ok = __all_sync(0xffffffffu, got);
            if (ok) {
                const uint8_t *src = smem + (g ? L::kDO : L::kQ) + row * 128;
                uint32_t rv[D / 2];
#pragma unroll
                for (int c = 0; c < D / 64; ++c)
#pragma unroll
                    for (int k16 = 0; k16 < 8; ++k16) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(src + c * L::kChunkBytes + ((k16 ^ (row & 7)) * 16));
                        rv[c * 32 + 4 * k16 + 0] = u.x;
                        rv[c * 32 + 4 * k16 + 1] = u.y;
                        rv[c * 32 + 4 * k16 + 2] = u.z;
                        rv[c * 32 + 4 * k16 + 3] = u.w;
                    }
                if constexpr (D == 128)
                    tmem_st32dp_x64(tl + (g ? L::kColDO : L::kColQ), rv);
                else
                    tmem_st32dp_x32(tl + (g ? L::kColDO : L::kColQ), rv);
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(bar(L::kQDReady));
        }
        float lse2 = pos_inf(), di = 0.f;
        if (q < len_q) {
            const float l = __ldg(p.lse + sr.q_row0 + q);
            lse2 = (l == neg_inf()) ? pos_inf() : l * kLog2e;
            di = __ldg(p.Di + sr.q_row0 + q);
        }
        // last key this row may see
        const int lim = CAUSAL ? min(q + coff, len_k - 1) : len_k - 1;
        // this row of the general mask (rows past Nq read nothing)
        const float *mrow = nullptr;
        if (HAS_MASK && q < p.Nq)
            mrow = p.mask + (plane * p.Nq + q) * p.ldm;
        int kt = next_ktile<HAS_MASK>(p, plane, qt, 0, n_range);   // key tile of step j
        for (int j = 0; j < n && ok; ++j, kt = next_ktile<HAS_MASK>(p, plane, qt, kt + 1, n_range)) {
            const int kg = kt * kBK + 64 * g;                 // first key of this thread's half
            float mk[HAS_MASK ? 64 : 1];
            if constexpr (HAS_MASK) {
                // issued before the wait for S so the loads overlap it
                if (mrow != nullptr && kg + 64 <= p.Nk) {
                    const float4 *m4 = reinterpret_cast<const float4 *>(mrow + kg);
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float4 mm = __ldg(m4 + e);
                        mk[4 * e] = mm.x * kLog2e;
                        mk[4 * e + 1] = mm.y * kLog2e;
                        mk[4 * e + 2] = mm.z * kLog2e;
                        mk[4 * e + 3] = mm.w * kLog2e;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 64; ++e)
                        mk[e] = (mrow != nullptr && kg + e < p.Nk) ? __ldg(mrow + kg + e) * kLog2e : 0.f;
                }
            }
            {
                const bool got = mbar_wait(bar(L::kSFull), j & 1, wctx);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            }
            tc_fence_after();
            // ---- P = 2^(S qk + bias - LSE_2), kept in registers
            float pr[64];
            {
                uint32_t sv[64];
                tmem_ld32dp_x64_wait(tl + L::kColS + 64 * g, sv);
                tc_fence_before();
                mbar_arrive(bar(L::kSRead));   // the S columns may now be overwritten
                const float *bs = reinterpret_cast<const float *>(smem + L::kBias) +
                                  (j % L::kKStages) * 128 + 64 * g;
                const bool edge = kg + 63 > lim;
                const float2 qk2 = make_float2(qk, qk);
                const float2 nl2 = make_float2(-lse2, -lse2);
                // Without masked scores in this thread's columns, one pair in
                // kEmuEvery takes the FMA-pipe exponential instead of MUFU.
                auto make_p = [&](auto emu_tag) {
                    constexpr bool kEmu = decltype(emu_tag)::value;
#pragma unroll
                    for (int e = 0; e < 64; e += 2) {
                        const float2 sc = make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1]));
                        float2 x;
                        if constexpr (HAS_BIAS)
                            x = __ffma2_rn(sc, qk2, __fadd2_rn(make_float2(bs[e], bs[e + 1]), nl2));
                        else if constexpr (HAS_MASK)
                            x = __ffma2_rn(sc, qk2, __fadd2_rn(make_float2(mk[e], mk[e + 1]), nl2));
                        else
                            x = __ffma2_rn(sc, qk2, nl2);
                        if (!kEmu && edge) {
                            if (kg + e > lim) x.x = neg_inf();
                            if (kg + e + 1 > lim) x.y = neg_inf();
                        }
                        if (kEmu && (e / 2) % kEmuEvery == kEmuEvery - 1) {
                            const float2 pp = exp2_fma2(x);
                            pr[e] = pp.x;
                            pr[e + 1] = pp.y;
                        } else {
                            pr[e] = ex2_approx(x.x);
                            pr[e + 1] = ex2_approx(x.y);
                        }
                    }
                };
                if (__all_sync(0xffffffffu, !HAS_BIAS && !HAS_MASK && !edge && q < len_q))   // warp-uniform
                    make_p(std::true_type{});
                else
                    make_p(std::false_type{});
            }
            // ---- dS = P (dP - D), 16-bit, over the dP columns this thread read
            {
                const bool got = mbar_wait(bar(L::kDPFull), j & 1, wctx);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            }
            tc_fence_after();
            {
                uint32_t dpv[64];
                tmem_ld32dp_x64_wait(tl + L::kColDP + 64 * g, dpv);
                uint32_t dd[32];
                const float2 nd2 = make_float2(-di, -di);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float2 d = __fmul2_rn(make_float2(pr[2 * e], pr[2 * e + 1]),
                                                __fadd2_rn(make_float2(__uint_as_float(dpv[2 * e]), __uint_as_float(dpv[2 * e + 1])), nd2));
                    dd[e] = pack2<BF16>(d.x, d.y);
                }
                tmem_st32dp_x32(tl + L::kColDP + 64 * g, dd);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(L::kDSFull));
        }
        // ---- epilogue (warpgroup 0): dQ = scale * acc, 16-bit, staged in the Q buffer
        if (g != 0) ok = false;
        if (ok && n > 0) {
            const bool got = mbar_wait(bar(L::kOFull), 0, wctx);
            ok = __all_sync(0xffffffffu, got);
            tc_fence_after();
        }
        if (ok && VARLEN) {
            // packed sequences: each thread stores its own query row
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.dq) + (sr.q_row0 + q) * D);
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t v[32];
                if (n > 0) {
                    tmem_ld32dp_x32_wait(tl + L::kColDQ + cc * 32, v);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0u;
                }
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[e] = pack2<BF16>(__uint_as_float(v[2 * e]) * p.scale, __uint_as_float(v[2 * e + 1]) * p.scale);
                if (q < len_q) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        dst[cc * 4 + q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                }
            }
        } else if (ok) {
            uint8_t *stage = smem + L::kQ;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t v[32];
                if (n > 0) {
                    tmem_ld32dp_x32_wait(tl + L::kColDQ + cc * 32, v);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0u;
                }
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[e] = pack2<BF16>(__uint_as_float(v[2 * e]) * p.scale, __uint_as_float(v[2 * e + 1]) * p.scale);
                stage_row_sw128(stage, row, cc * 32, pk, L::kChunkBytes);
            }
            fence_proxy_async_smem();
            __syncwarp();
            const int row0 = q0 + wq * 32;
            if (lane == 0 && row0 < p.Nq) {
                for (int c = 0; c < D / 64; ++c)
                    tma_store_3d(&tm_dq, sbase + L::kQ + c * L::kChunkBytes + wq * 32 * 128, c * 64, row0, bh);
                tma_store_commit();
                tma_store_wait_all();
            }
        }
        tc_fence_before();
        named_bar_sync(1, kThreads);
    } else {
        named_bar_sync(1, kThreads);   // idle warps 10, 11
    }
}

template <int D, bool BF16, bool CAUSAL, bool HAS_BIAS, bool HAS_MASK = false, bool VARLEN = false>
cudaError_t launch_grad_t(const BwdTensorMaps &tm, const BwdParams &p, cudaStream_t stream) {
    {
        using L = DkdvLayout<D>;
        auto kern = fa_bwd_dkdv_kernel<D, BF16, CAUSAL, HAS_BIAS, HAS_MASK, VARLEN>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
        if (e != cudaSuccess) return e;
        const unsigned grid = static_cast<unsigned>((p.Nk + kBK - 1) / kBK) * p.B * p.H;
        prof_begin(stream, "fa_bwd_dkdv_kernel");
        kern<<<grid, kThreads, L::kBytes, stream>>>(tm.q, tm.k, tm.v, tm.dO, tm.dk, tm.dv, p);
        prof_end(stream);
        note_launch();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        using L = DqLayout<D>;
        auto kern = fa_bwd_dq_kernel<D, BF16, CAUSAL, HAS_BIAS, HAS_MASK, VARLEN>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
        if (e != cudaSuccess) return e;
        const unsigned grid = static_cast<unsigned>((p.Nq + kBQ - 1) / kBQ) * p.B * p.H;
        prof_begin(stream, "fa_bwd_dq_kernel");
        kern<<<grid, kThreads, L::kBytes, stream>>>(tm.q, tm.k, tm.v, tm.dO, tm.dq, p);
        prof_end(stream);
        note_launch();
        return cudaGetLastError();
    }
}

// 1. D_i = rowsum(dO * O) into the workspace (every row of the layout)
template <int D, bool BF16>
cudaError_t launch_pre(const BwdParams &p, cudaStream_t s) {
    const long long rows = p.cu_q ? static_cast<long long>(p.H) * p.total_q
                                  : static_cast<long long>(p.B) * p.H * p.Nq;
    constexpr long long kRowsPerBlock = 8LL * (32 / (D / 8)) * kPreUnroll;   // 8 warps per block
    const unsigned grid = static_cast<unsigned>(std::min<long long>((rows + kRowsPerBlock - 1) / kRowsPerBlock, 148LL * 8));
    prof_begin(s, "fa_bwd_pre_kernel");
    fa_bwd_pre_kernel<D, BF16><<<grid, 256, 0, s>>>(static_cast<const uint16_t *>(p.o),
                                                     static_cast<const uint16_t *>(p.dO), p.Di, rows);
    prof_end(s);
    note_launch();
    return cudaGetLastError();
}

template <int D, bool BF16>
cudaError_t launch_bwd_mask_d(const BwdTensorMaps &tm, const BwdParams &p, bool causal, cudaStream_t s) {
    cudaError_t e = launch_pre<D, BF16>(p, s);
    if (e != cudaSuccess) return e;
    return causal ? launch_grad_t<D, BF16, true, false, true>(tm, p, s)
                  : launch_grad_t<D, BF16, false, false, true>(tm, p, s);
}

template <int D, bool BF16>
cudaError_t launch_bwd_varlen_d(const BwdTensorMaps &tm, const BwdParams &p, bool causal, cudaStream_t s) {
    cudaError_t e = launch_pre<D, BF16>(p, s);
    if (e != cudaSuccess) return e;
    return causal ? launch_grad_t<D, BF16, true, false, false, true>(tm, p, s)
                  : launch_grad_t<D, BF16, false, false, false, true>(tm, p, s);
}

template <int D, bool BF16>
cudaError_t launch_bwd_d(const BwdTensorMaps &tm, const BwdParams &p, bool causal, bool bias,
                         cudaStream_t s) {
    // 1. D_i
    cudaError_t e = launch_pre<D, BF16>(p, s);
    if (e != cudaSuccess) return e;
    // 2. dK, dV and 3. dQ
    if (causal)
        return bias ? launch_grad_t<D, BF16, true, true>(tm, p, s) : launch_grad_t<D, BF16, true, false>(tm, p, s);
    return bias ? launch_grad_t<D, BF16, false, true>(tm, p, s) : launch_grad_t<D, BF16, false, false>(tm, p, s);
}

}  // namespace

cudaError_t launch_bwd_mask(const BwdTensorMaps &tm, const BwdParams &p, int D, bool bf16, bool causal,
                            cudaStream_t stream) {
    if (D == 64) return bf16 ? launch_bwd_mask_d<64, true>(tm, p, causal, stream)
                             : launch_bwd_mask_d<64, false>(tm, p, causal, stream);
    return bf16 ? launch_bwd_mask_d<128, true>(tm, p, causal, stream)
                : launch_bwd_mask_d<128, false>(tm, p, causal, stream);
}

cudaError_t launch_bwd_varlen(const BwdTensorMaps &tm, const BwdParams &p, int D, bool bf16, bool causal,
                              cudaStream_t stream) {
    if (D == 64) return bf16 ? launch_bwd_varlen_d<64, true>(tm, p, causal, stream)
                             : launch_bwd_varlen_d<64, false>(tm, p, causal, stream);
    return bf16 ? launch_bwd_varlen_d<128, true>(tm, p, causal, stream)
                : launch_bwd_varlen_d<128, false>(tm, p, causal, stream);
}

cudaError_t launch_bwd(const BwdTensorMaps &tm, const BwdParams &p, int D, bool bf16, bool causal,
                       bool has_bias, cudaStream_t stream) {
    if (D == 64) return bf16 ? launch_bwd_d<64, true>(tm, p, causal, has_bias, stream)
                             : launch_bwd_d<64, false>(tm, p, causal, has_bias, stream);
    return bf16 ? launch_bwd_d<128, true>(tm, p, causal, has_bias, stream)
                : launch_bwd_d<128, false>(tm, p, causal, has_bias, stream);
}

}  // namespace fa
