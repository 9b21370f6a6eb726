// fa_internal.h -- structures shared between the C-ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace fa {

// Storage types of Q, K, V (O is 16-bit: the input type, or bf16 for E4M3).
enum ElemType : int { kElemF16 = 0, kElemBF16 = 1, kElemE4M3 = 2 };

// Forward launch parameters (everything except the tensor maps).
struct FwdParams {
    int B, H, Nq, Nk;
    int n_mblocks;                 // ceil(Nq / 256): work units per (b, h)
    int n_units;                   // n_mblocks * B * H (* num_splits)
    int causal_off;                // Nk - Nq (bottom-right causal alignment)
    float qk_scale_log2;           // scale * log2(e) (E4M3: times the Q and K descales)
    float o_scale;                 // multiplies O = o / l at the end (E4M3: the V descale)
    const float *bias;             // [B, Nk] or nullptr
    const float *mask;             // [mask_B, mask_H, Nq, ldm] or nullptr
    int mask_B, mask_H;            // 1 (broadcast) or B, H
    long long ldm;                 // mask row stride (elements, multiple of 4, >= Nk)
    const uint8_t *tile_flags;     // [mask planes, ceil(Nq/128), ceil(Nk/128)] or nullptr
    // packed variable-length sequences (nullptr: fixed [B, H, N, D] layout).
    // Then Nq, Nk are the maxima of the sequence lengths, the tensors are
    // [H, total, D] and sequence b owns rows [cu_q[b], cu_q[b+1]) of q and o and
    // [cu_k[b], cu_k[b+1]) of k and v.
    const int *cu_q, *cu_k;
    int total_q, total_k;
    void *o;                       // [B*H, Nq, D] 16-bit output
    float *lse;                    // [B*H, Nq]
    int *err;                      // device error word
    unsigned long long timeout_ns; // limit of every device-side wait
    // split-KV only: key tiles [s * tiles_per_split, (s + 1) * tiles_per_split)
    int num_splits;
    int tiles_per_split;
    float *o_part;                 // [num_splits, B*H, Nq, D] fp32
    float *lse_part;               // [num_splits, B*H, Nq]
};

struct FwdTensorMaps {
    CUtensorMap q, k, v;
};

// Backward launch parameters.
struct BwdParams {
    int B, H, Nq, Nk;
    int causal_off;                // Nk - Nq
    float qk_scale_log2;           // scale * log2(e)
    float scale;
    const float *bias;             // [B, Nk] or nullptr
    const float *mask;             // [mask_B, mask_H, Nq, ldm] or nullptr
    int mask_B, mask_H;            // 1 (broadcast) or B, H
    long long ldm;                 // mask row stride (elements, multiple of 4, >= Nk)
    const uint8_t *tile_flags;     // [mask planes, ceil(Nq/128), ceil(Nk/128)] or nullptr
    const int *cu_q, *cu_k;        // packed variable-length sequences (see FwdParams)
    int total_q, total_k;
    const float *lse;              // [B*H, Nq] from the forward
    const void *o, *dO;            // [B*H, Nq, D] 16-bit
    void *dq, *dk, *dv;            // outputs (also written through tensor maps)
    float *Di;                     // workspace: [B*H*Nq] (packed: [H*total_q])
    int *err;
    unsigned long long timeout_ns;
};

struct BwdTensorMaps {
    CUtensorMap q, k, v, dO, dk, dv, dq;
};

cudaError_t launch_bwd(const BwdTensorMaps &tm, const BwdParams &p, int D, bool bf16, bool causal,
                       bool has_bias, cudaStream_t stream);
// Backward with the general additive mask p.mask (no key bias).
cudaError_t launch_bwd_mask(const BwdTensorMaps &tm, const BwdParams &p, int D, bool bf16, bool causal,
                            cudaStream_t stream);
// Backward of packed variable-length sequences (p.cu_q, p.cu_k).
cudaError_t launch_bwd_varlen(const BwdTensorMaps &tm, const BwdParams &p, int D, bool bf16, bool causal,
                              cudaStream_t stream);

// Rows of one (sequence, head) in the packed or fixed layout: the first row
// of its queries and keys in the [B*H or H, N or total, D] row space, and its
// lengths.
struct SeqRows {
    long long q_row0, k_row0;      // first q/o row and first k/v row of (b, h)
    int len_q, len_k;
};

__host__ __device__ inline SeqRows seq_rows(int bh, int H, int Nq, int Nk, const int *cu_q, const int *cu_k,
                                            int total_q, int total_k) {
    SeqRows r;
    if (cu_q == nullptr) {
        r.q_row0 = static_cast<long long>(bh) * Nq;
        r.k_row0 = static_cast<long long>(bh) * Nk;
        r.len_q = Nq;
        r.len_k = Nk;
    } else {
        // the table is read as given but clamped, so that no access can leave
        // [0, total) or exceed the maximum lengths whatever it holds
        const int b = bh / H, h = bh % H;
        const int q0 = min(max(cu_q[b], 0), total_q), k0 = min(max(cu_k[b], 0), total_k);
        r.q_row0 = static_cast<long long>(h) * total_q + q0;
        r.k_row0 = static_cast<long long>(h) * total_k + k0;
        r.len_q = min(max(cu_q[b + 1] - q0, 0), min(Nq, total_q - q0));
        r.len_k = min(max(cu_k[b + 1] - k0, 0), min(Nk, total_k - k0));
    }
    return r;
}

// Summary of a general mask: one byte per 128 x 128 tile of each plane, 1 if
// any entry of the tile is above -inf (fa_mask_tile_flags).
cudaError_t launch_mask_tile_flags(const float *mask, int planes, int Nq, int Nk, long long ldm,
                                   uint8_t *flags, cudaStream_t stream);

// Does the 128-row query tile qt of mask plane `plane` need key tile kt?
// (Without a summary every tile is needed.)
__host__ __device__ inline bool mask_tile_needed(const uint8_t *flags, long long plane, int Nq, int Nk, int qt,
                                                 int kt) {
    if (flags == nullptr) return true;
    const int n_qt = (Nq + 127) / 128, n_kt = (Nk + 127) / 128;
    if (qt < 0 || qt >= n_qt) return false;
    return flags[(plane * n_qt + qt) * n_kt + kt] != 0;
}

// Plane of the general mask used by head bh (b = bh / H, h = bh % H).
__host__ __device__ inline long long mask_plane(int bh, int H, int mask_B, int mask_H) {
    const int b = bh / H, h = bh % H;
    return static_cast<long long>(mask_B > 1 ? b : 0) * mask_H + (mask_H > 1 ? h : 0);
}

// Counts every kernel launch made by the library (fa_launch_count()).
void note_launch(unsigned n = 1);

// Per-kernel timing aid (fa_profile_enable / fa_profile_read): when enabled on
// the calling host thread, each launch is bracketed by two events on its stream.
void prof_begin(cudaStream_t stream, const char *name);
void prof_end(cudaStream_t stream);

// Persistent launches: `grid` CTAs (at most one per SM) take the p.n_units
// work units in a fixed snake order.
cudaError_t launch_fwd(const FwdTensorMaps &tm, const FwdParams &p, int D, int elem, bool causal,
                       bool has_bias, int grid, cudaStream_t stream);
// Forward with the general additive mask p.mask (16-bit inputs, no key bias).
cudaError_t launch_fwd_mask(const FwdTensorMaps &tm, const FwdParams &p, int D, bool bf16, bool causal,
                            int grid, cudaStream_t stream);
// Forward of packed variable-length sequences (p.cu_q, p.cu_k; 16-bit inputs).
cudaError_t launch_fwd_varlen(const FwdTensorMaps &tm, const FwdParams &p, int D, bool bf16, bool causal,
                              int grid, cudaStream_t stream);
cudaError_t launch_fwd_split(const FwdTensorMaps &tm, const FwdParams &p, int D, bool bf16, bool causal,
                             bool has_bias, int grid, cudaStream_t stream);
cudaError_t launch_fwd_empty(void *o, float *lse, size_t n_rows, int D, bool bf16,
                             cudaStream_t stream);

// Work-unit order of the backward recompute kernels (one CTA = one unit):
// heads in groups of kHeadGroup and, within a group, tile-major with the
// heaviest tile rank first.  The CTAs in flight at any time then share the
// streamed Q/dO (or K/V) tiles of a few heads in L2 instead of all heads',
// and across the grid the long causal units still start before the short
// ones.  Maps idx in [0, n_heads * n_tiles) one-to-one onto
// (tile_rank, head); the caller turns tile_rank 0 into its heaviest tile.
#ifdef __CUDACC__
__device__ __forceinline__ void unit_of(int idx, int n_heads, int n_tiles, int &tile_rank, int &head) {
    constexpr int kHeadGroup = 8;
    const int per_group = kHeadGroup * n_tiles;
    const int grp = idx / per_group;
    const int r = idx - grp * per_group;
    const int g0 = grp * kHeadGroup;
    const int gsz = min(kHeadGroup, n_heads - g0);
    tile_rank = r / gsz;
    head = g0 + r % gsz;
}
#endif

}  // namespace fa
