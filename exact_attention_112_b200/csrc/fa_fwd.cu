// fa_fwd.cu -- fused exact-attention forward for sm_100a (B200).
//
// What it computes: O = softmax(scale * Q K^T + mask) V and the row
// log-sum-exp, as defined on the FlashAttention case-study slides
// (nmj0.github.io, "Attention is where tokens meet"), organised as on the
// slide "FlashAttention: the idea": Q, K, V are cut into tiles that fit on
// chip, QK^T, mask, softmax and .V of a tile run in one kernel, and neither S
// nor P is ever written to device memory.  Tiles are combined with the running
// (m, l, o) update of "Online softmax: divide once, at the end"; O = o / l is
// formed once per row after the last tile.
//
// B200 mapping.  A work unit is 256 query rows (two 128-row tensor-core tiles
// Q0, Q1) of one (batch, head), optionally restricted to one range of key
// tiles (split-KV).  The kernel is persistent: one CTA per SM takes the units
// in a fixed order (heaviest first -- the causal units that see the most key
// tiles -- dealt out in a snake over the CTAs, which balances the causal
// triangle as well as a greedy longest-first schedule), so tensor memory,
// barriers and the pipeline are set up once per SM and the next unit's Q load
// and first S products overlap the current unit's epilogue.
//   * TMA streams Q (two tiles per unit, each released as soon as its last S
//     product has read it; the next unit's Q is prefetched into L2 when the
//     current unit starts) and K_j / V_j through a 2-stage shared-memory
//     ring that runs on across unit boundaries, each stage handed over by an
//     mbarrier (expect_tx / complete_tx).
//   * The MMA warp issues tcgen05.mma from one elected lane while the whole
//     warp runs the loop (warp-uniform descriptors and counters): S_i =
//     Q_i K_j^T (both operands from shared memory, fp32 accumulator in tensor
//     memory) and O_i += P_i V_j (P_i read from tensor memory, V_j from shared
//     memory).  16-bit inputs use kind::f16 (K = 16 per instruction); E4M3
//     inputs use kind::f8f6f4 (K = 32) with P rounded to E4M3.
//   * Two softmax warpgroups (one per Q tile, one thread per query row) read
//     S_i from tensor memory, apply scale and mask in the base-2 domain
//     (qk_scale = scale * log2(e), the constant derived in "Mastering
//     FlashAttention: The Algebraic Foundation"), update the row max and sum in
//     registers and write P_i back over the S_i columns in two halves of 64
//     keys, each with its own barrier, so the first half of P_i V_j runs while
//     the second half is still being exponentiated.  Three exponentials in
//     four run on the MUFU unit, the fourth on the FMA pipe (exp2_fma2).
//   * Lazy rescale: the reference maximum m_ref of a row only moves when a new
//     tile's maximum exceeds it by more than kTau (log2 units); only then are
//     l and the O accumulator multiplied by alpha = 2^(m_ref_old - m_ref_new).
//     Exactness rests on the slide's identity e^(s - m_old) e^(m_old - m_new)
//     = e^(s - m_new): l, o and the final LSE all use the same m_ref.
//   * Causal: key tiles entirely above the diagonal are never loaded or
//     multiplied; tiles crossing it are masked per element.
//   * Additive terms after scaling: a per-key bias [B, Nk] (copied one key
//     tile ahead into a shared-memory slot per warp and read as broadcasts),
//     or a general mask [B or 1, H or 1, Nq, Nk] whose row each softmax
//     thread reads itself (the "+ mask" of the SDPA formula in full).
//   * Epilogue: each softmax thread divides its O row by l and stores it
//     straight from registers (so the Q buffer is free for the next unit).
//
// MMA issue order (one in-order tensor pipe): per key tile t of a unit
//     PV_0(t) [half 0, half 1], S_0(t+1), PV_1(t) [half 0, half 1], S_1(t+1)
// and at a unit boundary PV_0(t), PV_1(t), S_0(next), S_1(next).
//
// Tensor memory (512 columns x 128 lanes of 32 bits; lane = query row):
//   cols [0,128)        S_0 (fp32), then P_0 over its first 64 (16-bit) or 32 (E4M3) columns
//   cols [128,256)      S_1 / P_1
//   cols [256,256+D)    O_0 accumulator (fp32)
//   cols [256+D,256+2D) O_1 accumulator
// Shared memory: Q_0, Q_1, K ring x2, V ring x2, mbarriers.
//
// Warp roles (12 warps): 0-3 softmax of Q_0, 4-7 softmax of Q_1, 8 TMA
// producer, 9 MMA issuer (also allocates tensor memory), 10-11 idle (they
// only complete the third warpgroup for the register split).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <type_traits>

#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

constexpr int kBM = 128;            // query rows per tensor-core tile
constexpr int kBN = 128;            // keys per tile
constexpr int kThreads = 384;       // 12 warps = three warpgroups
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
// Register split (launch pool 168 x 384 = 64512): the two softmax warpgroups
// take 192 each, the producer/MMA warpgroup (warps 8-11, 10-11 idle) 120:
// 8*32*192 + 4*32*120 = 64512; per SMSP (192 + 192 + 120) * 32 = 16128 <= 16384.
constexpr uint32_t kRegsSoftmax = 192;
constexpr uint32_t kRegsOther = 120;
constexpr int kStages = 2;
constexpr float kTau = 8.0f;        // lazy-rescale threshold (log2 units)
constexpr int kEmuEvery = 4;        // one pair of exponentials in kEmuEvery on the FMA pipe
constexpr float kLn2 = 0.69314718055994530942f;

template <int D, int ELEM>
struct FwdLayout {
    static constexpr int kElemBytes = ELEM == kElemE4M3 ? 1 : 2;
    static constexpr int kRowBytes = D * kElemBytes;      // one Q/K/V row
    static constexpr int kChunkElems = 128 / kElemBytes;  // values per 128-byte swizzle row
    static constexpr int kChunks = kRowBytes / 128;       // 128-byte column blocks per row
    static constexpr int kTileBytes = kBM * kRowBytes;    // one 128-row tile
    static constexpr int kChunkBytes = kBM * 128;         // 128 rows x 128 bytes
    static constexpr int kKSteps = kRowBytes / 32;        // MMA K-steps of S (32 bytes each)
    static constexpr int kPvKeys = 32 / kElemBytes;       // keys per P.V instruction
    static constexpr int kPvSteps = kBN / kPvKeys;        // P.V instructions per tile
    static constexpr int kQ = 0;                          // 2 tiles
    static constexpr int kK = kQ + 2 * kTileBytes;        // kStages tiles
    static constexpr int kV = kK + kStages * kTileBytes;  // kStages tiles
    static constexpr int kBar = kV + kStages * kTileBytes;
    // barrier indices
    static constexpr int kQFull = 0;     // +tile
    static constexpr int kQEmpty = 2;    // +tile
    static constexpr int kKFull = 4;     // +stage
    static constexpr int kKEmpty = 6;    // +stage
    static constexpr int kVFull = 8;     // +stage
    static constexpr int kVEmpty = 10;   // +stage
    static constexpr int kSFull = 12;    // +tile
    static constexpr int kPHalf = 14;    // +2*tile+half
    static constexpr int kOFull = 18;    // +tile
    static constexpr int kDrain = 20;
    static constexpr int kNumBars = 21;
    static constexpr int kMisc = kBar + kNumBars * 8;  // tmem base, abort flag
    // per softmax warp: two slots of one key tile of bias (fp32)
    static constexpr int kBiasStage = (kMisc + 16 + 15) / 16 * 16;
    static constexpr int kBiasSlot = kBN * 4;
    static constexpr int kBytes = kBiasStage + 8 * 2 * kBiasSlot;
    static constexpr int kAlloc = kBytes + 1024;       // room to align the base
    static constexpr int kAllocNoBias = kBiasStage + 1024;   // kernels without a key bias
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
    static_assert(kChunks >= 1 && kRowBytes % 128 == 0, "rows must be whole 128-byte swizzle rows");
    static_assert(kAlloc <= 232448, "shared memory");
    static_assert(kBiasStage % 16 == 0, "float4 bias slots");
};

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

// 32 bytes to global memory in one 256-bit store (sm_100); `p` must be 32-byte
// aligned.  A row-per-thread store then fills whole 32-byte sectors instead of
// halves of two.
__device__ __forceinline__ void st_global_v8(void *p, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t a4, uint32_t a5, uint32_t a6, uint32_t a7) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a0), "r"(a1),
                 "r"(a2), "r"(a3), "r"(a4), "r"(a5), "r"(a6), "r"(a7)
                 : "memory");
}

// Two fp32 values -> one 32-bit word of two 16-bit values (lo in the low half).
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

// Four fp32 values -> one 32-bit word of four E4M3 values (a in the low byte),
// round to nearest even, saturating at the largest finite E4M3 value.
__device__ __forceinline__ uint32_t pack4_e4m3(float a, float b, float c, float d) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
    return lo | (hi << 16);
}

// One work unit: rows [m0, m0 + 256) of head bh (rows counted within the
// head's sequence), key tiles [kv_first, kv_first + n_kv) (n_kv == 0: the
// rows see no key).  The sequence has len_q queries and len_k keys; its rows
// sit at y = q_y0 + row (k_y0 + key) of the tensor maps' head slice z, and
// its O / LSE rows start at o_row0.
struct Unit {
    int bh, m0, kv_first, n_kv, split;
    int len_q, len_k, q_y0, k_y0, z;
    long long o_row0;
    // with a general mask and its tile summary, the unit visits only the key
    // tiles in [kv_first, kv_end) that the summary marks for one of its two
    // query tiles; n_kv counts those
    int kv_end;
    long long plane;
};

// First key tile k >= from of the unit that must be visited (kv_end if none).
template <bool HAS_MASK>
__device__ __forceinline__ int next_tile(const FwdParams &p, const Unit &w, int from) {
    if constexpr (HAS_MASK) {
        if (p.tile_flags != nullptr) {
            const int qt0 = w.m0 / kBM;
            for (int k = from; k < w.kv_end; ++k)
                if (mask_tile_needed(p.tile_flags, w.plane, p.Nq, p.Nk, qt0, k) ||
                    mask_tile_needed(p.tile_flags, w.plane, p.Nq, p.Nk, qt0 + 1, k))
                    return k;
            return w.kv_end;
        }
    }
    return from;
}

template <bool CAUSAL, bool SPLIT, bool VARLEN = false, bool HAS_MASK = false>
__device__ __forceinline__ Unit unit_info(const FwdParams &p, int u) {
    Unit w;
    const int BH = p.B * p.H;
    w.split = 0;
    if (SPLIT) {
        w.split = u % p.num_splits;
        u /= p.num_splits;
    }
    // heaviest (last) query blocks first
    const int mb = (p.n_mblocks - 1) - u / BH;
    w.bh = u % BH;
    w.m0 = mb * 2 * kBM;
    if constexpr (VARLEN) {
        const SeqRows sr = seq_rows(w.bh, p.H, p.Nq, p.Nk, p.cu_q, p.cu_k, p.total_q, p.total_k);
        w.z = w.bh % p.H;
        w.len_q = sr.len_q;
        w.len_k = sr.len_k;
        w.q_y0 = static_cast<int>(sr.q_row0 - static_cast<long long>(w.z) * p.total_q);
        w.k_y0 = static_cast<int>(sr.k_row0 - static_cast<long long>(w.z) * p.total_k);
        w.o_row0 = sr.q_row0;
    } else {
        w.len_q = p.Nq;
        w.len_k = p.Nk;
        w.q_y0 = 0;
        w.k_y0 = 0;
        w.z = w.bh;
        w.o_row0 = static_cast<long long>(w.bh) * p.Nq;
    }
    const int n_kv_all = (w.len_k + kBN - 1) / kBN;
    w.n_kv = w.m0 < w.len_q ? n_kv_all : 0;   // a block past the sequence's end has no rows
    if (CAUSAL && w.n_kv > 0) {
        const int last_row = min(w.m0 + 2 * kBM - 1, w.len_q - 1);
        const int lim = last_row + (w.len_k - w.len_q);
        w.n_kv = lim < 0 ? 0 : min(n_kv_all, lim / kBN + 1);
    }
    w.kv_first = 0;
    if (SPLIT) {
        w.kv_first = w.split * p.tiles_per_split;
        w.n_kv = max(0, min(w.n_kv, w.kv_first + p.tiles_per_split) - w.kv_first);
    }
    w.kv_end = w.kv_first + w.n_kv;
    w.plane = 0;
    if constexpr (HAS_MASK) {
        w.plane = mask_plane(w.bh, p.H, p.mask_B, p.mask_H);
        if (p.tile_flags != nullptr) {
            int n = 0;
            for (int k = next_tile<true>(p, w, w.kv_first); k < w.kv_end; k = next_tile<true>(p, w, k + 1)) ++n;
            w.n_kv = n;
        }
    }
    return w;
}

// r-th unit of this CTA in the snake order, or -1 when it has no more.
__device__ __forceinline__ int unit_at(const FwdParams &p, int r) {
    const int G = gridDim.x;
    const long long u = static_cast<long long>(r) * G + ((r & 1) ? (G - 1 - static_cast<int>(blockIdx.x)) : blockIdx.x);
    return u < p.n_units ? static_cast<int>(u) : -1;
}

// Advance r to this CTA's next unit that has key tiles (the producer and the
// MMA warp skip the others); false when none is left.
template <bool CAUSAL, bool SPLIT, bool VARLEN = false, bool HAS_MASK = false>
__device__ __forceinline__ bool next_work(const FwdParams &p, int &r, Unit &w) {
    for (;; ++r) {
        const int u = unit_at(p, r);
        if (u < 0) return false;
        w = unit_info<CAUSAL, SPLIT, VARLEN, HAS_MASK>(p, u);
        if (w.n_kv > 0) return true;
    }
}

template <int D, int ELEM, bool CAUSAL, bool HAS_BIAS, bool SPLIT = false, bool HAS_MASK = false,
          bool VARLEN = false>
__global__ void __launch_bounds__(kThreads, 1)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using L = FwdLayout<D, ELEM>;
    // scores arrive already scaled (and offset) when an additive term is present
    constexpr bool kAdd = HAS_BIAS || HAS_MASK;
    constexpr bool kFp8 = ELEM == kElemE4M3;
    constexpr bool kOutBF16 = ELEM != kElemF16;   // O storage type
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    auto bar = [&](int i) -> uint32_t { return sbase + L::kBar + 8 * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int BH = p.B * p.H;

    // ---- set-up (once per CTA)
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(L::kQFull + i), 1);
            mbar_init(bar(L::kQEmpty + i), 1);
            mbar_init(bar(L::kSFull + i), 1);
            mbar_init(bar(L::kPHalf + 2 * i), 4 * 32);
            mbar_init(bar(L::kPHalf + 2 * i + 1), 4 * 32);
            mbar_init(bar(L::kOFull + i), 1);
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(L::kKFull + s), 1);
            mbar_init(bar(L::kKEmpty + s), 1);
            mbar_init(bar(L::kVFull + s), 1);
            mbar_init(bar(L::kVEmpty + s), 1);
        }
        mbar_init(bar(L::kDrain), 1);
        fence_mbar_init();
    }
    if (warp == kProducerWarp && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtx wctx{p.timeout_ns, p.err, abort_flag};
    // Register split: warpgroup 2 (producer, MMA, two idle warps) gives
    // registers back, the softmax warpgroups take them.  Nobody asks for
    // registers again afterwards, so the split cannot deadlock; every role ends
    // in its own branch at the CTA barrier 1, and the MMA warp frees tensor
    // memory after it.
    if (warp >= 8) regs_release<kRegsOther>();
    if (warp == kProducerWarp) {
        // ===================== TMA producer =====================
        if (lane == 0) {
            bool ok = true;
            int t = 0;          // key tiles loaded so far (ring position)
            int uc = 0;         // units with key tiles started so far
            int kv_half = 0;    // K and V loads issued (2 per key tile)
            int q_issued = 0;   // Q tiles issued for the current unit
            int r = 0;
            Unit w;
            while (ok && next_work<CAUSAL, SPLIT, VARLEN, HAS_MASK>(p, r, w)) {
                // Q_i of this unit, once the previous unit's last S_i has read Q_i
                q_issued = 0;
                for (int i = 0; i < 2 && ok; ++i) {
                    if (uc > 0 && !mbar_wait(bar(L::kQEmpty + i), (uc - 1) & 1, wctx)) { ok = false; break; }
                    mbar_arrive_expect_tx(bar(L::kQFull + i), L::kTileBytes);
                    for (int c = 0; c < L::kChunks; ++c)
                        tma_load_3d(sbase + L::kQ + i * L::kTileBytes + c * L::kChunkBytes, &tm_q,
                                    bar(L::kQFull + i), c * L::kChunkElems, w.q_y0 + w.m0 + i * kBM, w.z);
                    q_issued = i + 1;
                }
                if (!ok) break;
                {   // warm L2 with the next unit's Q tiles while this unit runs; a
                    // unit of fewer than 8 key tiles does without (measured: the
                    // prefetch then delays more than it hides)
                    int r2 = r + 1;
                    Unit nx;
                    if (w.n_kv >= 8 && next_work<CAUSAL, SPLIT, VARLEN, HAS_MASK>(p, r2, nx))
                        for (int i = 0; i < 2; ++i)
                            for (int c = 0; c < L::kChunks; ++c)
                                tma_prefetch_l2_3d(&tm_q, c * L::kChunkElems, nx.q_y0 + nx.m0 + i * kBM, nx.z);
                }
                int kt = next_tile<HAS_MASK>(p, w, w.kv_first);      // key tile of step j
                for (int j = 0; j < w.n_kv; ++j, ++t, kt = next_tile<HAS_MASK>(p, w, kt + 1)) {
                    const int s = t & 1;
                    const uint32_t ph = (t >> 1) & 1;
                    const int row = w.k_y0 + kt * kBN;
                    if (!mbar_wait(bar(L::kKEmpty + s), ph ^ 1, wctx)) { ok = false; break; }
                    mbar_arrive_expect_tx(bar(L::kKFull + s), L::kTileBytes);
                    for (int c = 0; c < L::kChunks; ++c)
                        tma_load_3d(sbase + L::kK + s * L::kTileBytes + c * L::kChunkBytes, &tm_k,
                                    bar(L::kKFull + s), c * L::kChunkElems, row, w.z);
                    ++kv_half;
                    if (!mbar_wait(bar(L::kVEmpty + s), ph ^ 1, wctx)) { ok = false; break; }
                    mbar_arrive_expect_tx(bar(L::kVFull + s), L::kTileBytes);
                    for (int c = 0; c < L::kChunks; ++c)
                        tma_load_3d(sbase + L::kV + s * L::kTileBytes + c * L::kChunkBytes, &tm_v,
                                    bar(L::kVFull + s), c * L::kChunkElems, row, w.z);
                    ++kv_half;
                }
                if (!ok) break;
                ++uc;
                ++r;
            }
            if (!ok) {
                // Give the copies already in flight a bounded chance to land
                // before the CTA (and its shared memory) goes away.
                WaitCtx drain{wctx.timeout_ns, wctx.err, nullptr};
                volatile int zero = 0;
                drain.abort_flag = &zero;
                for (int i = 0; i < q_issued; ++i) mbar_wait(bar(L::kQFull + i), uc & 1, drain);
                for (int h = (kv_half > 4 ? kv_half - 4 : 0); h < kv_half; ++h) {
                    const int tt = h >> 1;
                    mbar_wait(bar(((h & 1) ? L::kVFull : L::kKFull) + (tt & 1)), (tt >> 1) & 1, drain);
                }
            }
        }
        named_bar_sync(1, kThreads);
    } else if (warp == kMmaWarp) {
        // ============ MMA issuer (whole warp; one elected lane issues) ============
        int r = 0;
        Unit w;
        const bool have = next_work<CAUSAL, SPLIT, VARLEN, HAS_MASK>(p, r, w);
        if (have) {
            constexpr uint32_t idesc_qk = kFp8 ? idesc_e4m3_f32acc(kBM, kBN, false, false)
                                               : idesc_f16_f32acc(ELEM == kElemBF16, kBM, kBN, false, false);
            constexpr uint32_t idesc_pv = kFp8 ? idesc_e4m3_f32acc(kBM, D, false, true)
                                               : idesc_f16_f32acc(ELEM == kElemBF16, kBM, D, false, true);
            // S_i = Q_i K^T into the S_i columns; commits s_full(i), then
            // k_empty(stage) after S_1, then q_empty(i) after a unit's last S_i
            auto issue_s = [&](int i, int stage, bool release_k, bool release_q) {
                const uint64_t dq = smem_desc_sw128(sbase + L::kQ + i * L::kTileBytes, 16, 1024);
                const uint64_t dk = smem_desc_sw128(sbase + L::kK + stage * L::kTileBytes, 16, 1024);
                const uint32_t d = tmem + (i ? L::kColS1 : L::kColS0);
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < L::kKSteps; ++kk) {
                        const uint32_t off = ((kk >> 2) * L::kChunkBytes + (kk & 3) * 32) >> 4;
                        if constexpr (kFp8)
                            umma_f8_ss(d, dq + off, dk + off, idesc_qk, kk > 0);
                        else
                            umma_f16_ss(d, dq + off, dk + off, idesc_qk, kk > 0);
                    }
                    umma_commit(bar(L::kSFull + i));
                    if (release_k) umma_commit(bar(L::kKEmpty + stage));
                    if (release_q) umma_commit(bar(L::kQEmpty + i));
                }
                __syncwarp();
            };
            // O_i += P_i V (A: P_i over the S_i columns), K-steps [k0, k1)
            auto issue_pv = [&](int i, int stage, bool acc, int k0, int k1) {
                const uint64_t dv = smem_desc_sw128(sbase + L::kV + stage * L::kTileBytes, L::kChunkBytes, 1024);
                const uint32_t pa = tmem + (i ? L::kColS1 : L::kColS0);
                const uint32_t d = tmem + (i ? L::kColO1 : L::kColO0);
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < L::kPvSteps; ++kk) {
                        if (kk < k0 || kk >= k1) continue;
                        const uint64_t b = dv + ((kk * L::kPvKeys * 128) >> 4);
                        if constexpr (kFp8)
                            umma_f8_ts(d, pa + kk * 8, b, idesc_pv, (acc || kk > 0) ? 1u : 0u);
                        else
                            umma_f16_ts(d, pa + kk * 8, b, idesc_pv, (acc || kk > 0) ? 1u : 0u);
                    }
                }
                __syncwarp();
            };
            auto commit = [&](uint32_t b) {
                if (elect_one()) umma_commit(b);
                __syncwarp();
            };
            constexpr int kHalf = L::kPvSteps / 2;
            int t = 0;      // key tiles issued so far (ring position, S/P barrier phases)
            int uc = 0;     // units done so far (Q and O barrier phases)
            bool ok = mbar_wait_warp(bar(L::kQFull + 0), 0, wctx) && mbar_wait_warp(bar(L::kKFull + 0), 0, wctx);
            if (ok) {
                tc_fence_after();
                issue_s(0, 0, false, w.n_kv == 1);
                ok = mbar_wait_warp(bar(L::kQFull + 1), 0, wctx);
            }
            if (ok) {
                tc_fence_after();
                issue_s(1, 0, true, w.n_kv == 1);
            }
            while (ok) {
                for (int j = 0; j < w.n_kv && ok; ++j, ++t) {
                    const int s = t & 1;
                    const uint32_t ph = (t >> 1) & 1;
                    const bool last = j + 1 == w.n_kv;
                    int r2 = r + 1;
                    Unit nx = w;
                    const bool has_next = !last || next_work<CAUSAL, SPLIT, VARLEN, HAS_MASK>(p, r2, nx);
                    const int s1 = (t + 1) & 1;
                    const uint32_t ph1 = ((t + 1) >> 1) & 1;
                    const uint32_t pp = t & 1;
                    if (!mbar_wait_warp(bar(L::kVFull + s), ph, wctx)) { ok = false; break; }
                    // ---- P_0 V(t), half by half
                    if (!mbar_wait_warp(bar(L::kPHalf + 0), pp, wctx)) { ok = false; break; }
                    tc_fence_after();
                    issue_pv(0, s, j > 0, 0, kHalf);
                    if (!mbar_wait_warp(bar(L::kPHalf + 1), pp, wctx)) { ok = false; break; }
                    tc_fence_after();
                    issue_pv(0, s, j > 0, kHalf, L::kPvSteps);
                    if (last) commit(bar(L::kOFull + 0));
                    // ---- S_0(t+1) inside the unit
                    if (!last) {
                        if (!mbar_wait_warp(bar(L::kKFull + s1), ph1, wctx)) { ok = false; break; }
                        tc_fence_after();
                        issue_s(0, s1, false, j + 2 == w.n_kv);
                    }
                    // ---- P_1 V(t)
                    if (!mbar_wait_warp(bar(L::kPHalf + 2), pp, wctx)) { ok = false; break; }
                    tc_fence_after();
                    issue_pv(1, s, j > 0, 0, kHalf);
                    if (!mbar_wait_warp(bar(L::kPHalf + 3), pp, wctx)) { ok = false; break; }
                    tc_fence_after();
                    issue_pv(1, s, j > 0, kHalf, L::kPvSteps);
                    commit(bar(L::kVEmpty + s));
                    if (last) commit(bar(L::kOFull + 1));
                    // ---- S_1(t+1), or both S products of the next unit's first tile
                    if (has_next) {
                        if (last) {
                            if (!mbar_wait_warp(bar(L::kQFull + 0), (uc + 1) & 1, wctx) ||
                                !mbar_wait_warp(bar(L::kKFull + s1), ph1, wctx)) { ok = false; break; }
                            tc_fence_after();
                            issue_s(0, s1, false, nx.n_kv == 1);
                            if (!mbar_wait_warp(bar(L::kQFull + 1), (uc + 1) & 1, wctx)) { ok = false; break; }
                            tc_fence_after();
                            issue_s(1, s1, true, nx.n_kv == 1);
                        } else {
                            issue_s(1, s1, true, j + 2 == w.n_kv);
                        }
                    }
                }
                if (!ok) break;
                ++uc;
                ++r;
                if (!next_work<CAUSAL, SPLIT, VARLEN, HAS_MASK>(p, r, w)) break;
            }
        }
        if (have) {
            // Every issued MMA must finish before tensor memory is released.
            if (elect_one()) umma_commit(bar(L::kDrain));
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
        // ===================== softmax warpgroups =====================
        regs_alloc<kRegsSoftmax>();
        const int i = warp >> 2;            // which Q tile
        const int wq = warp & 3;            // lane quarter of tensor memory
        const int row = wq * 32 + lane;     // row within the tile (= TMEM lane)
        const uint32_t tl = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        const uint32_t tS = tl + (i ? L::kColS1 : L::kColS0);
        const uint32_t tO = tl + (i ? L::kColO1 : L::kColO0);
        const float qk = p.qk_scale_log2;
        // O rows start on 128-byte multiples of the base: 256-bit stores when
        // the base is 32-byte aligned (the library asks for 16 only)
        const bool o_v8 = (reinterpret_cast<uintptr_t>(p.o) & 31) == 0;
        // Key bias: every row of a tile adds the same 128 values.  Each warp
        // copies them (cp.async, four per lane) into its own shared-memory slot
        // one tile ahead, scales them by log2(e) in place when the tile starts,
        // and the tile reads them as broadcasts.  Two slots alternate by tile.
        uint8_t *bslots = smem + L::kBiasStage + warp * 2 * L::kBiasSlot;
        auto bias_fetch = [&](const float *bias_b, int kv0, int slot) {
            const int c0 = kv0 + 4 * lane;
            const float *src = bias_b + c0;
            const uint32_t dst = smem_u32(bslots + slot * L::kBiasSlot + 16 * lane);
            if ((reinterpret_cast<uintptr_t>(bias_b) & 15) == 0 && (p.Nk & 3) == 0) {
                const int n = min(max(p.Nk - c0, 0), 4);
                cp_async_zfill<16>(dst, n > 0 ? src : bias_b, 4 * n);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const bool in = c0 + e < p.Nk;
                    cp_async_zfill<4>(dst + 4 * e, in ? src + e : bias_b, in ? 4 : 0);
                }
            }
        };
        bool ok = true;
        int t = 0;      // key tiles seen so far (S/P barrier phases)
        int uc = 0;     // units with key tiles done so far (O barrier phase)
        for (int r = 0; ok; ++r) {
            const int u = unit_at(p, r);
            if (u < 0) break;
            const Unit w = unit_info<CAUSAL, SPLIT, VARLEN, HAS_MASK>(p, u);
            const int qrow = w.m0 + i * kBM + row;   // within the head's sequence
            // last key index this row may see
            const int lim = CAUSAL ? min(qrow + (w.len_k - w.len_q), w.len_k - 1) : w.len_k - 1;
            const float *bias_b = HAS_BIAS ? p.bias + static_cast<size_t>(w.bh / p.H) * p.Nk : nullptr;
            if constexpr (HAS_BIAS) {
                if (w.n_kv > 0) bias_fetch(bias_b, next_tile<HAS_MASK>(p, w, w.kv_first) * kBN, t & 1);
                cp_async_commit();
            }
            // this row of the general mask (rows past Nq read nothing)
            const float *mrow = nullptr;
            if (HAS_MASK && qrow < w.len_q)
                mrow = p.mask + (mask_plane(w.bh, p.H, p.mask_B, p.mask_H) * p.Nq + qrow) * p.ldm;
            float m_ref = neg_inf();   // log2 units
            float l = 0.f;
            int kt = next_tile<HAS_MASK>(p, w, w.kv_first);          // key tile of step j
            for (int j = 0; j < w.n_kv; ++j, ++t, kt = next_tile<HAS_MASK>(p, w, kt + 1)) {
                const int kv0 = kt * kBN;
                if constexpr (HAS_BIAS) {
                    // every lane has finished reading the other slot (previous
                    // tile) before it is refilled with the next tile's bias
                    __syncwarp();
                    if (j + 1 < w.n_kv) bias_fetch(bias_b, next_tile<HAS_MASK>(p, w, kt + 1) * kBN, (t + 1) & 1);
                    cp_async_commit();
                    cp_async_wait<1>();          // this tile's copy has landed
                    float4 *mine = reinterpret_cast<float4 *>(bslots + (t & 1) * L::kBiasSlot) + lane;
                    constexpr float kLog2e = 1.4426950408889634f;
                    const float4 b = *mine;
                    *mine = make_float4(b.x * kLog2e, b.y * kLog2e, b.z * kLog2e, b.w * kLog2e);
                    __syncwarp();
                }
                {
                    const bool got = mbar_wait(bar(L::kSFull + i), t & 1, wctx);
                    if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                }
                tc_fence_after();
                uint32_t sr[128];
                tmem_ld32dp_x128_wait(tS, sr);
                float x[128];
                if constexpr (HAS_BIAS) {
                    // x = s * qk_scale + bias * log2(e), the bias from this warp's
                    // slot (columns past Nk hold 0 and are masked below)
                    const float4 *bt = reinterpret_cast<const float4 *>(bslots + (t & 1) * L::kBiasSlot);
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const float4 bb = bt[c];
                        x[4 * c + 0] = fmaf(__uint_as_float(sr[4 * c + 0]), qk, bb.x);
                        x[4 * c + 1] = fmaf(__uint_as_float(sr[4 * c + 1]), qk, bb.y);
                        x[4 * c + 2] = fmaf(__uint_as_float(sr[4 * c + 2]), qk, bb.z);
                        x[4 * c + 3] = fmaf(__uint_as_float(sr[4 * c + 3]), qk, bb.w);
                    }
                } else if constexpr (HAS_MASK) {
                    // x = s * qk_scale + M_ij * log2(e); the thread reads its own
                    // row (512 contiguous bytes per tile, L1-cached)
                    constexpr float kLog2e = 1.4426950408889634f;
                    if (mrow != nullptr && kv0 + kBN <= p.Nk) {
                        const float4 *m4 = reinterpret_cast<const float4 *>(mrow + kv0);
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const float4 mm = __ldg(m4 + c);
                            x[4 * c + 0] = fmaf(__uint_as_float(sr[4 * c + 0]), qk, mm.x * kLog2e);
                            x[4 * c + 1] = fmaf(__uint_as_float(sr[4 * c + 1]), qk, mm.y * kLog2e);
                            x[4 * c + 2] = fmaf(__uint_as_float(sr[4 * c + 2]), qk, mm.z * kLog2e);
                            x[4 * c + 3] = fmaf(__uint_as_float(sr[4 * c + 3]), qk, mm.w * kLog2e);
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 128; ++c) {
                            const float mm = (mrow != nullptr && kv0 + c < p.Nk) ? __ldg(mrow + kv0 + c) * kLog2e : 0.f;
                            x[c] = fmaf(__uint_as_float(sr[c]), qk, mm);
                        }
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 128; ++c) x[c] = __uint_as_float(sr[c]);
                }
                if (kv0 + kBN - 1 > lim) {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (kv0 + c > lim) x[c] = neg_inf();
                }
                // row maximum: four independent chains of three-input maxima
                float mx0 = x[0], mx1 = x[1], mx2 = x[2], mx3 = x[3];
#pragma unroll
                for (int c = 4; c < 124; c += 8) {
                    mx0 = fmax3(mx0, x[c], x[c + 1]);
                    mx1 = fmax3(mx1, x[c + 2], x[c + 3]);
                    mx2 = fmax3(mx2, x[c + 4], x[c + 5]);
                    mx3 = fmax3(mx3, x[c + 6], x[c + 7]);
                }
                float m_tile = fmax3(fmax3(mx0, mx1, x[124]), fmax3(mx2, mx3, x[125]), fmaxf(x[126], x[127]));
                if constexpr (!kAdd) m_tile *= qk;   // qk > 0: max commutes with scaling
                const bool need = m_tile > m_ref + kTau;
                // warp-uniform: if any row of the warp moves its reference maximum,
                // the warp rescales its O rows (before the first half of P is
                // handed over, below)
                const bool rescale = __any_sync(0xffffffffu, need);
                float alpha = 1.f;
                if (rescale) {
                    const float m_new = need ? m_tile : m_ref;
                    alpha = (m_ref == neg_inf()) ? 0.f : ex2_approx(m_ref - m_new);
                    l *= alpha;
                    m_ref = m_new;
                }
                const float m_use = (m_ref == neg_inf()) ? 0.f : m_ref;
                // p = 2^(x - m), two columns per paired-fp32 instruction, in two
                // halves of 64 keys; each half goes back over the S columns and
                // is handed to the MMA warp on its own barrier.  One pair in
                // kEmuEvery goes through the FMA-pipe exponential instead of MUFU
                // once every row of the warp has a finite reference maximum: a
                // masked score (-inf) then yields 2^-126 instead of 0, which is
                // invisible next to l >= 1 (the score that set m_ref contributes
                // 2^(m_tile - m_ref) >= 1); rows that have seen no key yet keep
                // the exact MUFU path so that they still end with l = 0.
                float2 lsum = make_float2(0.f, 0.f), lsum2 = make_float2(0.f, 0.f);
                const float2 neg_m2 = make_float2(-m_use, -m_use);
                const float2 qk2 = make_float2(qk, qk);
                const bool emu = __all_sync(0xffffffffu, m_ref != neg_inf());   // warp-uniform
                auto half = [&](int h, auto emu_tag) {
                    constexpr bool kEmu = decltype(emu_tag)::value;
                    float pv[64];
#pragma unroll
                    for (int c2 = 0; c2 < 32; ++c2) {
                        const int c = 64 * h + 2 * c2;
                        const float2 xc = make_float2(x[c], x[c + 1]);
                        const float2 a = kAdd ? __fadd2_rn(xc, neg_m2) : __ffma2_rn(xc, qk2, neg_m2);
                        float2 pp;
                        if (kEmu && c2 % kEmuEvery == kEmuEvery - 1)
                            pp = exp2_fma2(a);
                        else
                            pp = make_float2(ex2_approx(a.x), ex2_approx(a.y));
                        if (c2 & 1)
                            lsum2 = __fadd2_rn(lsum2, pp);
                        else
                            lsum = __fadd2_rn(lsum, pp);
                        pv[2 * c2] = pp.x;
                        pv[2 * c2 + 1] = pp.y;
                    }
                    if constexpr (kFp8) {
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            pk[e] = pack4_e4m3(pv[4 * e], pv[4 * e + 1], pv[4 * e + 2], pv[4 * e + 3]);
                        tmem_st32dp_x16(tS + 16 * h, pk);
                    } else {
                        uint32_t pk[32];
#pragma unroll
                        for (int e = 0; e < 32; ++e) pk[e] = pack2<ELEM == kElemBF16>(pv[2 * e], pv[2 * e + 1]);
                        tmem_st32dp_x32(tS + 32 * h, pk);
                    }
                };
                if (emu)
                    half(0, std::true_type{});
                else
                    half(0, std::false_type{});
                if (rescale && j > 0) {
                    // O_i row *= alpha.  O is stable: the MMA that produced this
                    // S tile was issued after the previous P.V and its commit
                    // covers it; the next P.V waits for the arrive below.
#pragma unroll
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t orr[32];
                        tmem_ld32dp_x32_wait(tO + cc * 32, orr);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
                        tmem_st32dp_x32(tO + cc * 32, orr);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(L::kPHalf + 2 * i));
                if (emu)
                    half(1, std::true_type{});
                else
                    half(1, std::false_type{});
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(L::kPHalf + 2 * i + 1));
                l += (lsum.x + lsum.y) + (lsum2.x + lsum2.y);
            }
            if (!ok) break;

            // ---- epilogue: O = o / l (times o_scale), LSE = (m_ref + log2 l) ln 2
            if (w.n_kv > 0) {
                const bool got = mbar_wait(bar(L::kOFull + i), uc & 1, wctx);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                tc_fence_after();
                ++uc;
            }
            const float inv_l = l > 0.f ? p.o_scale / l : 0.f;
            const float lse = l > 0.f ? (m_ref + lg2_approx(l)) * kLn2 : neg_inf();
            if (SPLIT) {
                // partial result of this key range: O_s = o / l (fp32), LSE_s
                const size_t prow = (static_cast<size_t>(w.split) * BH + w.bh) * p.Nq + qrow;
                static_assert(!(SPLIT && VARLEN), "split-KV partials use the fixed layout");
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t orr[32];
                    if (w.n_kv > 0) {
                        tmem_ld32dp_x32_wait(tO + cc * 32, orr);
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) orr[e] = 0u;
                    }
                    if (qrow < p.Nq) {
                        float4 *dst = reinterpret_cast<float4 *>(p.o_part + prow * D + cc * 32);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            dst[e] = make_float4(__uint_as_float(orr[4 * e]) * inv_l, __uint_as_float(orr[4 * e + 1]) * inv_l,
                                                 __uint_as_float(orr[4 * e + 2]) * inv_l, __uint_as_float(orr[4 * e + 3]) * inv_l);
                    }
                }
                if (qrow < p.Nq) p.lse_part[prow] = lse;
            } else {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.o) +
                                                       (w.o_row0 + qrow) * D);
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t orr[32];
                    if (w.n_kv > 0) {
                        tmem_ld32dp_x32_wait(tO + cc * 32, orr);
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) orr[e] = 0u;
                    }
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = pack2<kOutBF16>(__uint_as_float(orr[2 * e]) * inv_l,
                                                __uint_as_float(orr[2 * e + 1]) * inv_l);
                    if (qrow < w.len_q) {
                        if (o_v8) {
                            // whole 32-byte sectors per store instruction
#pragma unroll
                            for (int h8 = 0; h8 < 2; ++h8)
                                st_global_v8(dst + cc * 4 + 2 * h8, pk[8 * h8], pk[8 * h8 + 1], pk[8 * h8 + 2],
                                             pk[8 * h8 + 3], pk[8 * h8 + 4], pk[8 * h8 + 5], pk[8 * h8 + 6],
                                             pk[8 * h8 + 7]);
                        } else {
#pragma unroll
                            for (int q4 = 0; q4 < 4; ++q4)
                                dst[cc * 4 + q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                        }
                    }
                }
                if (qrow < w.len_q) p.lse[w.o_row0 + qrow] = lse;
            }
            // the next unit's first P.V may overwrite O_i only after these loads
            tc_fence_before();
        }
        if constexpr (HAS_BIAS) cp_async_wait<0>();   // no bias copy outlives the CTA
        named_bar_sync(1, kThreads);
    } else {
        named_bar_sync(1, kThreads);   // idle warps 10, 11
    }
}

// Merge of the split-KV partials, one warp per query row:
//   LSE = m + ln sum_s exp(LSE_s - m),  O = sum_s exp(LSE_s - m) O_s / sum_s exp(LSE_s - m)
// with m = max_s LSE_s (all -inf: the row saw no key, O = 0, LSE = -inf).
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_fwd_combine_kernel(const float *__restrict__ o_part,
                                                             const float *__restrict__ lse_part,
                                                             uint16_t *__restrict__ o, float *__restrict__ lse,
                                                             long long rows, int num_splits) {
    constexpr int kPer = D / 32;   // values per lane (2 or 4)
    constexpr int kU = 4;          // O_s rows in flight per lane
    const int lane = threadIdx.x & 31;
    const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    for (long long r = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows; r += nwarps) {
        // m = max_s LSE_s, the lanes taking the splits in turn
        float m = neg_inf();
        for (int sp = lane; sp < num_splits; sp += 32) m = fmaxf(m, lse_part[sp * rows + r]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        float acc[kPer];
#pragma unroll
        for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
        float wsum = 0.f;
        if (m != neg_inf()) {
            for (int s0 = 0; s0 < num_splits; s0 += 32) {
                // lane k holds the weight of split s0 + k; every lane sums the
                // weighted O_s rows of the chunk, kU loads in flight
                float wl = 0.f;
                if (s0 + lane < num_splits) {
                    const float ls = lse_part[(s0 + lane) * rows + r];
                    wl = ls == neg_inf() ? 0.f : __expf(ls - m);
                }
                wsum += wl;
                const int cnt = min(32, num_splits - s0);
                for (int k = 0; k < cnt; k += kU) {
                    float w[kU], v[kU][kPer];
#pragma unroll
                    for (int u = 0; u < kU; ++u) {
                        w[u] = __shfl_sync(0xffffffffu, wl, (k + u) & 31);
                        const int sp = s0 + min(k + u, cnt - 1);
                        const float *src = o_part + (sp * rows + r) * D + lane * kPer;
                        if constexpr (kPer == 4) {
                            const float4 t4 = *reinterpret_cast<const float4 *>(src);
                            v[u][0] = t4.x; v[u][1] = t4.y; v[u][2] = t4.z; v[u][3] = t4.w;
                        } else {
                            const float2 t2 = *reinterpret_cast<const float2 *>(src);
                            v[u][0] = t2.x; v[u][1] = t2.y;
                        }
                    }
#pragma unroll
                    for (int u = 0; u < kU; ++u) {
                        // a split that saw no key (weight 0) adds nothing, whatever its row holds
                        if (k + u < cnt && w[u] != 0.f) {
#pragma unroll
                            for (int e = 0; e < kPer; ++e) acc[e] = fmaf(w[u], v[u][e], acc[e]);
                        }
                    }
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
        }
        const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
        uint32_t packed[kPer / 2];
#pragma unroll
        for (int e = 0; e < kPer / 2; ++e) packed[e] = pack2<BF16>(acc[2 * e] * inv, acc[2 * e + 1] * inv);
        uint16_t *dst = o + r * D + lane * kPer;
        if constexpr (kPer == 4)
            *reinterpret_cast<uint2 *>(dst) = make_uint2(packed[0], packed[1]);
        else
            *reinterpret_cast<uint32_t *>(dst) = packed[0];
        if (lane == 0) lse[r] = wsum > 0.f ? m + __logf(wsum) : neg_inf();
    }
}

// Tile summary of a general mask: flags[plane][qt][kt] = 1 if any entry of the
// 128 x 128 tile (query rows qt*128.., keys kt*128..) is above -inf.  One
// block per tile; each warp reads whole 128-value row segments (coalesced).
__global__ void __launch_bounds__(128) fa_mask_flags_kernel(const float *__restrict__ mask, int Nq, int Nk,
                                                            long long ldm, uint8_t *__restrict__ flags) {
    const int kt = blockIdx.x, qt = blockIdx.y;
    const long long plane = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k0 = kt * 128 + lane * 4;
    bool any = false;
    for (int r = warp; r < 128; r += 4) {
        const int q = qt * 128 + r;
        if (q >= Nq) break;
        const float *row = mask + (plane * Nq + q) * ldm;
        if (k0 + 3 < Nk) {
            const float4 m = __ldg(reinterpret_cast<const float4 *>(row + k0));
            any |= m.x > neg_inf() || m.y > neg_inf() || m.z > neg_inf() || m.w > neg_inf();
        } else {
            for (int e = 0; e < 4; ++e)
                if (k0 + e < Nk) any |= __ldg(row + k0 + e) > neg_inf();
        }
    }
    const int hit = __syncthreads_or(any ? 1 : 0);
    if (threadIdx.x == 0)
        flags[(plane * gridDim.y + qt) * gridDim.x + kt] = hit ? 1 : 0;
}

// Rows with no key at all (Nk == 0): O = 0, LSE = -inf.
template <typename T>
__global__ void fa_fwd_empty_kernel(T *o, float *lse, size_t n_rows, int D) {
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    for (size_t r = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; r < n_rows; r += stride) {
        lse[r] = __int_as_float(0xff800000);
        for (int d = 0; d < D; ++d) o[r * D + d] = T(0.f);
    }
}

template <int D, int ELEM, bool CAUSAL, bool HAS_BIAS>
cudaError_t launch_fwd_t(const FwdTensorMaps &tm, const FwdParams &p, int grid, cudaStream_t stream) {
    using L = FwdLayout<D, ELEM>;
    auto kern = fa_fwd_kernel<D, ELEM, CAUSAL, HAS_BIAS>;
    constexpr int kSmem = HAS_BIAS ? L::kAlloc : L::kAllocNoBias;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    prof_begin(stream, "fa_fwd_kernel");
    kern<<<static_cast<unsigned>(grid), kThreads, kSmem, stream>>>(tm.q, tm.k, tm.v, p);
    prof_end(stream);
    note_launch();
    return cudaGetLastError();
}

template <int D, bool BF16, bool CAUSAL>
cudaError_t launch_mask_t(const FwdTensorMaps &tm, const FwdParams &p, int grid, cudaStream_t stream) {
    constexpr int kElem = BF16 ? kElemBF16 : kElemF16;
    using L = FwdLayout<D, kElem>;
    auto kern = fa_fwd_kernel<D, kElem, CAUSAL, false, false, true>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAllocNoBias);
    if (e != cudaSuccess) return e;
    prof_begin(stream, "fa_fwd_mask_kernel");
    kern<<<static_cast<unsigned>(grid), kThreads, L::kAllocNoBias, stream>>>(tm.q, tm.k, tm.v, p);
    prof_end(stream);
    note_launch();
    return cudaGetLastError();
}

template <int D, bool BF16, bool CAUSAL>
cudaError_t launch_varlen_t(const FwdTensorMaps &tm, const FwdParams &p, int grid, cudaStream_t stream) {
    constexpr int kElem = BF16 ? kElemBF16 : kElemF16;
    using L = FwdLayout<D, kElem>;
    auto kern = fa_fwd_kernel<D, kElem, CAUSAL, false, false, false, true>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAllocNoBias);
    if (e != cudaSuccess) return e;
    prof_begin(stream, "fa_fwd_varlen_kernel");
    kern<<<static_cast<unsigned>(grid), kThreads, L::kAllocNoBias, stream>>>(tm.q, tm.k, tm.v, p);
    prof_end(stream);
    note_launch();
    return cudaGetLastError();
}

template <int D, bool BF16, bool CAUSAL, bool HAS_BIAS>
cudaError_t launch_split_t(const FwdTensorMaps &tm, const FwdParams &p, int grid, cudaStream_t stream) {
    constexpr int kElem = BF16 ? kElemBF16 : kElemF16;
    using L = FwdLayout<D, kElem>;
    auto kern = fa_fwd_kernel<D, kElem, CAUSAL, HAS_BIAS, true>;
    constexpr int kSmem = HAS_BIAS ? L::kAlloc : L::kAllocNoBias;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    prof_begin(stream, "fa_fwd_split_kernel");
    kern<<<static_cast<unsigned>(grid), kThreads, kSmem, stream>>>(tm.q, tm.k, tm.v, p);
    prof_end(stream);
    note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const long long rows = static_cast<long long>(p.B) * p.H * p.Nq;
    const unsigned cgrid = static_cast<unsigned>(std::min<long long>((rows + 7) / 8, 148LL * 16));
    prof_begin(stream, "fa_fwd_combine_kernel");
    fa_fwd_combine_kernel<D, BF16><<<cgrid, 256, 0, stream>>>(p.o_part, p.lse_part, static_cast<uint16_t *>(p.o),
                                                               p.lse, rows, p.num_splits);
    prof_end(stream);
    note_launch();
    return cudaGetLastError();
}

template <int D, bool BF16>
cudaError_t launch_split_d(const FwdTensorMaps &tm, const FwdParams &p, bool causal, bool bias, int grid,
                           cudaStream_t s) {
    if (causal) return bias ? launch_split_t<D, BF16, true, true>(tm, p, grid, s) : launch_split_t<D, BF16, true, false>(tm, p, grid, s);
    return bias ? launch_split_t<D, BF16, false, true>(tm, p, grid, s) : launch_split_t<D, BF16, false, false>(tm, p, grid, s);
}

template <int D, int ELEM>
cudaError_t launch_fwd_d(const FwdTensorMaps &tm, const FwdParams &p, bool causal, bool bias, int grid,
                         cudaStream_t s) {
    if (causal) return bias ? launch_fwd_t<D, ELEM, true, true>(tm, p, grid, s) : launch_fwd_t<D, ELEM, true, false>(tm, p, grid, s);
    return bias ? launch_fwd_t<D, ELEM, false, true>(tm, p, grid, s) : launch_fwd_t<D, ELEM, false, false>(tm, p, grid, s);
}

}  // namespace

cudaError_t launch_fwd(const FwdTensorMaps &tm, const FwdParams &p, int D, int elem, bool causal,
                       bool has_bias, int grid, cudaStream_t stream) {
    if (elem == kElemE4M3) return launch_fwd_d<128, kElemE4M3>(tm, p, causal, has_bias, grid, stream);
    if (D == 64) return elem == kElemBF16 ? launch_fwd_d<64, kElemBF16>(tm, p, causal, has_bias, grid, stream)
                                          : launch_fwd_d<64, kElemF16>(tm, p, causal, has_bias, grid, stream);
    return elem == kElemBF16 ? launch_fwd_d<128, kElemBF16>(tm, p, causal, has_bias, grid, stream)
                             : launch_fwd_d<128, kElemF16>(tm, p, causal, has_bias, grid, stream);
}

cudaError_t launch_fwd_mask(const FwdTensorMaps &tm, const FwdParams &p, int D, bool bf16, bool causal,
                            int grid, cudaStream_t stream) {
    if (D == 64) {
        if (bf16) return causal ? launch_mask_t<64, true, true>(tm, p, grid, stream) : launch_mask_t<64, true, false>(tm, p, grid, stream);
        return causal ? launch_mask_t<64, false, true>(tm, p, grid, stream) : launch_mask_t<64, false, false>(tm, p, grid, stream);
    }
    if (bf16) return causal ? launch_mask_t<128, true, true>(tm, p, grid, stream) : launch_mask_t<128, true, false>(tm, p, grid, stream);
    return causal ? launch_mask_t<128, false, true>(tm, p, grid, stream) : launch_mask_t<128, false, false>(tm, p, grid, stream);
}

cudaError_t launch_fwd_varlen(const FwdTensorMaps &tm, const FwdParams &p, int D, bool bf16, bool causal,
                              int grid, cudaStream_t stream) {
    if (D == 64) {
        if (bf16) return causal ? launch_varlen_t<64, true, true>(tm, p, grid, stream) : launch_varlen_t<64, true, false>(tm, p, grid, stream);
        return causal ? launch_varlen_t<64, false, true>(tm, p, grid, stream) : launch_varlen_t<64, false, false>(tm, p, grid, stream);
    }
    if (bf16) return causal ? launch_varlen_t<128, true, true>(tm, p, grid, stream) : launch_varlen_t<128, true, false>(tm, p, grid, stream);
    return causal ? launch_varlen_t<128, false, true>(tm, p, grid, stream) : launch_varlen_t<128, false, false>(tm, p, grid, stream);
}

cudaError_t launch_fwd_split(const FwdTensorMaps &tm, const FwdParams &p, int D, bool bf16, bool causal,
                             bool has_bias, int grid, cudaStream_t stream) {
    if (D == 64) return bf16 ? launch_split_d<64, true>(tm, p, causal, has_bias, grid, stream)
                             : launch_split_d<64, false>(tm, p, causal, has_bias, grid, stream);
    return bf16 ? launch_split_d<128, true>(tm, p, causal, has_bias, grid, stream)
                : launch_split_d<128, false>(tm, p, causal, has_bias, grid, stream);
}

cudaError_t launch_mask_tile_flags(const float *mask, int planes, int Nq, int Nk, long long ldm, uint8_t *flags,
                                   cudaStream_t stream) {
    const dim3 grid((Nk + 127) / 128, (Nq + 127) / 128, planes);
    if (grid.x == 0 || grid.y == 0) return cudaSuccess;
    prof_begin(stream, "fa_mask_flags_kernel");
    fa_mask_flags_kernel<<<grid, 128, 0, stream>>>(mask, Nq, Nk, ldm, flags);
    prof_end(stream);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_fwd_empty(void *o, float *lse, size_t n_rows, int D, bool bf16, cudaStream_t stream) {
    const unsigned grid = static_cast<unsigned>(std::min<size_t>((n_rows + 255) / 256, 4096));
    if (grid == 0) return cudaSuccess;
    prof_begin(stream, "fa_fwd_empty_kernel");
    if (bf16)
        fa_fwd_empty_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(static_cast<__nv_bfloat16 *>(o), lse, n_rows, D);
    else
        fa_fwd_empty_kernel<__half><<<grid, 256, 0, stream>>>(static_cast<__half *>(o), lse, n_rows, D);
    prof_end(stream);
    note_launch();
    return cudaGetLastError();
}

}  // namespace fa
