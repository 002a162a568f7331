// schedule.cuh -- split-KV work distribution shared by the main and combine
// kernels (device side; computed from the lengths that live on the device, so
// a run needs no host synchronisation and can be captured in a CUDA graph).
//
// The KV tiles (kTileKV rows each) of all sequences are laid end to end:
// sequence b owns tiles [acc_b, acc_b + n_b) of a flat index space of N_t
// tiles.  The space is cut into P equal contiguous ranges of T = ceil(N_t/P)
// tiles ("partitions"); partition p is processed by one CTA (or CTA pair) per
// query-row group.  A sequence that falls inside one partition is finished by
// that CTA; a sequence cut by partition boundaries leaves one fp32 partial
// (O / l and its log-sum-exp) per piece, merged by the combine kernel.
//
// Partial slots: partition p owns slots 2p and 2p+1.  The piece of sequence b
// in partition p uses slot 2p if b started before p, else slot 2p+1 (b starts
// in p and continues after it).  Both can occur in one partition, for two
// different sequences; a sequence that both starts before and ends after p is
// p's only sequence and uses 2p.
#pragma once

#include <cstdint>

namespace mla {

constexpr int kTileKV = 128;       // kv rows per pipeline tile
constexpr int kDqk = 576;          // 512 latent + 64 rope
constexpr int kDv = 512;
constexpr int kChunk = 64;         // columns per 128-byte swizzled chunk
constexpr int kNumChunks = kDqk / kChunk;  // 9

// status word bits (workspace header, word 0)
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusSeqlen = 2u;

__device__ __forceinline__ int clamp_len(int L, int L_max, uint32_t* status) {
    if (L < 0 || L > L_max) {
        if (status) atomicOr(status, kStatusSeqlen);
        L = L < 0 ? 0 : L_max;
    }
    return L;
}

__device__ __forceinline__ int num_tiles(int L) { return (L + kTileKV - 1) / kTileKV; }

// Warp-cooperative: total tiles over all sequences, and (for `start`) the
// first sequence whose tiles reach past `start` with its flat offset.
// Every lane returns the same values.
struct ScanResult {
    long long total;     // N_t
    int b_first;         // first sequence with acc_b + n_b > start (or B)
    long long acc_first; // acc of b_first
};

__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ inline long long total_tiles_warp(const int32_t* seqlens, int B, int L_max) {
    const int lane = threadIdx.x & 31;
    long long s = 0;
    for (int b = lane; b < B; b += 32) s += num_tiles(clamp_len(seqlens[b], L_max, nullptr));
    return warp_sum_ll(s);
}

// Locate the first sequence overlapping flat tile `start` (warp-cooperative).
__device__ inline void locate_warp(const int32_t* seqlens, int B, int L_max, long long start, int* b_out,
                                   long long* acc_out) {
    const int lane = threadIdx.x & 31;
    long long acc = 0;
    for (int base = 0; base < B; base += 32) {
        const int b = base + lane;
        const long long n = (b < B) ? num_tiles(clamp_len(seqlens[b], L_max, nullptr)) : 0;
        // inclusive prefix within the warp
        long long incl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const long long excl = incl - n;
        // sequences with n > 0 whose range [acc+excl, acc+incl) reaches past start
        const bool hit = (b < B) && (n > 0) && (acc + incl > start);
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m) {
            const int src = __ffs(m) - 1;
            const long long e = __shfl_sync(0xffffffffu, excl, src);
            *b_out = base + src;
            *acc_out = acc + e;
            return;
        }
        acc += __shfl_sync(0xffffffffu, incl, 31);
    }
    *b_out = B;
    *acc_out = acc;
}

struct Piece {
    int b;          // sequence
    int L;          // its (clamped) length
    int tile_lo;    // first tile (sequence-local index)
    int tile_hi;    // one past the last tile
    int slot;       // partial slot, or -1 when the piece is the whole sequence
};

// Sequential walker over the pieces of one partition; every role of a CTA
// runs its own copy and sees the same sequence of pieces.
struct PieceWalker {
    const int32_t* seqlens;
    int B, L_max, p;
    long long start, end;  // flat tile range of this partition
    int b;                 // next sequence to look at
    long long acc;         // its flat offset

    __device__ bool next(Piece& out) {
        while (b < B && acc < end) {
            const int L = clamp_len(seqlens[b], L_max, nullptr);
            const long long n = num_tiles(L);
            const long long lo = acc > start ? acc : start;
            const long long hi = (acc + n) < end ? (acc + n) : end;
            const int cur = b;
            const long long acc_cur = acc;
            ++b;
            acc += n;
            if (hi <= lo) continue;
            out.b = cur;
            out.L = L;
            out.tile_lo = static_cast<int>(lo - acc_cur);
            out.tile_hi = static_cast<int>(hi - acc_cur);
            const bool starts_before = acc_cur < start;
            const bool continues_after = acc_cur + n > end;
            if (!starts_before && !continues_after) out.slot = -1;
            else out.slot = starts_before ? 2 * p : 2 * p + 1;
            return true;
        }
        return false;
    }
};

}  // namespace mla
