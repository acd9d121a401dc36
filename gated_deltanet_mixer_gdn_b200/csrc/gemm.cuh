// Dense bf16 GEMM on 5th-generation tensor cores for the projections around
// the mixer (module tree of the Qwen3.8 27B architecture page, `linear_attn`:
// in_proj_qkv 10240x5120, in_proj_z 6144x5120, in_proj_b / in_proj_a 48x5120,
// out_proj 5120x6144):
//     C[m][n] = sum_k A[m][k] W[n][k]       A [M][K], W [N][K] bf16, f32 accumulation
// with the columns of C routed to up to four output tensors (in_proj writes
// qkv, z, b and a from one product over the stacked weights).
//
// Persistent CTAs walk 128 x 256 output tiles (grouped: 16 M tiles swept across
// all N tiles, so a round's operands stay in L2).  One warp issues the TMA loads of A and
// W K-slices (64 wide, 128B swizzle) into a 4-stage ring, one warp issues
// tcgen05.mma (M = 128, N = 256, bf16) into one of two TMEM accumulators, and
// four warps drain the other accumulator (tcgen05.ld, round to bf16, store)
// while the next tile is multiplied.  The fused instance (FUSED = 1, see
// inproj.cuh) runs the mixer's load stage in that epilogue instead of storing
// the projection.
#pragma once

#include "common.cuh"

namespace gdn {

struct GemmSegment {
    int col0;        // first column of C this segment takes
    int ld;          // row stride of the destination (elements)
    uint16_t* dst;   // bf16 destination; segment column c lands at dst[row * ld + c - col0]
};

struct GemmParams {
    int M, N, K;
    int nseg;              // 1..4 segments, ascending col0, segment 0 at column 0
    GemmSegment seg[4];
};

// The load stage fused into the in_proj epilogue (see inproj.cuh).
struct FusedPrep {
    int Kh, Vh, T;                 // dense rows of T tokens (cu == nullptr)
    const int* cu;                 // packed rows: cu_seqlens [N+1] (device), or nullptr
    int N;                         // packed rows
    const uint16_t* conv_w;        // bf16 [C][4]
    const float* A_log;            // [Vh]
    const float* dt_bias;          // [Vh]
    const float* init_conv;        // f32 [rows][3][C] or nullptr
    __half *Qs, *Ks, *Ql, *Kl, *Vs;
    float *Gs, *Bs;                // [Vh][M]
    uint16_t* z;                   // bf16 [M][Vh*128]
    float* conv_last;              // f32 [rows][3][C]: pre-conv values of each row's last three tokens
                                   // (token pos of a row of len tokens in slot pos + 3 - len)
};

namespace gemm {
constexpr int BM = 128, BN = 256, BK = 64, kStages = 4;
constexpr uint32_t A_BYTES = BM * BK * 2;  // 16 KB
constexpr uint32_t B_BYTES = BN * BK * 2;  // 32 KB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t OFF_MISC = kStages * STAGE_BYTES;
constexpr int kXStride = 36;  // floats per row of the epilogue's exchange buffer (32 + 4: no bank conflicts)
constexpr uint32_t XBUF_BYTES = BM * kXStride * 4;       // 32 columns of every tile row
constexpr uint32_t SCRATCH_BYTES = XBUF_BYTES + 256 * 16;  // + the tile's conv taps as f32
constexpr uint32_t SMEM_BYTES = OFF_MISC + 256 + SCRATCH_BYTES + 1024;
constexpr int kThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr uint32_t TMEM_COLS = 512;  // two 256-column accumulators
// bf16 A and B (format 1), f32 accumulator, both K-major, M = 128, N = 256
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                           (static_cast<uint32_t>(BM >> 4) << 24);
// barriers: full[kStages], empty[kStages], acc_full[2], acc_empty[2]
constexpr int B_FULL = 0, B_EMPTY = kStages, B_ACCF = 2 * kStages, B_ACCE = 2 * kStages + 2;
}  // namespace gemm

// Tile t of the walk -> (M tile, N tile).  Groups of kGroupM M tiles are swept across all
// N tiles, M-fastest inside the group: a round of the persistent grid then touches about
// kGroupM row blocks of A and ~148 / kGroupM weight tiles, a working set that stays in L2,
// instead of streaming all of A for every weight tile.
constexpr int kGroupM = 32;
__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int& tm, int& tn) {
    const int per_group = kGroupM * tiles_n;
    const int g = t / per_group;
    const int r = t - g * per_group;
    const int gm = min(kGroupM, tiles_m - g * kGroupM);
    tn = r / gm;
    tm = g * kGroupM + (r - tn * gm);
}

template <int FUSED>
__device__ void fused_prep_epilogue(const FusedPrep& f, const GemmParams& p, uint32_t tacc, int r0, int n0,
                                    uint8_t* scratch, int q4, int lane);

// FUSED = 0: plain C = A W^T.  FUSED = 1: in_proj with the load stage in the
// epilogue; M tiles then start 3 rows early (each 128-row tile yields 125
// tokens whose conv window lies inside the tile).
template <int FUSED>
__global__ void __launch_bounds__(gemm::kThreads, 1)
    gdn_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                    const GemmParams p, const FusedPrep f) {
    using namespace gemm;
    constexpr int kStepM = FUSED ? BM - 3 : BM;  // tokens per M tile
    constexpr int kLead = FUSED ? 3 : 0;        // rows of the tile before its first output token
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_MISC);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + OFF_MISC + 128);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tiles_m = (p.M + kStepM - 1) / kStepM, tiles_n = (p.N + BN - 1) / BN;
    const int ntiles = tiles_m * tiles_n;
    const int ksteps = p.K / BK;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars[B_FULL + s], 1);
            mbar_init(&bars[B_EMPTY + s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars[B_ACCF + b], 1);
            mbar_init(&bars[B_ACCE + b], 4);  // one arrive per epilogue warp
        }
        fence_barrier_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmW);
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem;
    bool broken = false;
    auto wait1 = [&](int slot, uint32_t parity) {
        if (!broken && !mbar_wait(&bars[slot], parity)) {
            broken = true;
            record_error(kErrTimeoutTma);
        }
    };

    if (warp == 0) {
        // ---------------- TMA: K-slices of A and W into the ring
        if (lane == 0) {
            uint32_t q = 0;  // ring position over all tiles
            for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
                int tm, tn;
                tile_coords(t, tiles_m, tiles_n, tm, tn);
                const int m0 = tm * kStepM - kLead, n0 = tn * BN;  // m0 < 0: zero rows
                for (int ks = 0; ks < ksteps; ++ks, ++q) {
                    const int s = q % kStages;
                    if (q >= kStages) wait1(B_EMPTY + s, ((q / kStages) - 1) & 1);
                    uint8_t* st = smem + s * STAGE_BYTES;
                    mbar_arrive_expect_tx(&bars[B_FULL + s], STAGE_BYTES);
                    tma_load_2d(st, &tmA, ks * BK, m0, &bars[B_FULL + s]);
                    tma_load_2d(st + A_BYTES, &tmW, ks * BK, n0, &bars[B_FULL + s]);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issue
        if (lane == 0) {
            uint32_t q = 0, it = 0;
            for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
                const int ab = it & 1;
                if (it >= 2) wait1(B_ACCE + ab, ((it >> 1) - 1) & 1);  // the epilogue drained this accumulator
                tc_fence_after();
                const uint32_t d = tbase + ab * BN;
                for (int ks = 0; ks < ksteps; ++ks, ++q) {
                    const int s = q % kStages;
                    wait1(B_FULL + s, (q / kStages) & 1);
                    tc_fence_after();
                    const uint32_t aA = sbase + s * STAGE_BYTES, aW = aA + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_f16(d, sw128_desc(aA + kk * 32, 16, 1024), sw128_desc(aW + kk * 32, 16, 1024), IDESC,
                                (ks > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&bars[B_EMPTY + s]);  // the stage may be refilled once these MMAs are done
                }
                mma_commit(&bars[B_ACCF + ab]);
            }
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: TMEM -> bf16 -> the output segments
        const int q4 = warp & 3;  // TMEM lane quarter of this warp
        const uint32_t tl = static_cast<uint32_t>(32 * q4) << 16;
        uint32_t it = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
            const int ab = it & 1;
            int tm, tn;
            tile_coords(t, tiles_m, tiles_n, tm, tn);
            const int m0 = tm * kStepM - kLead, n0 = tn * BN;
            wait1(B_ACCF + ab, (it >> 1) & 1);
            __syncwarp();
            tc_fence_after();
            if constexpr (FUSED != 0) {
                fused_prep_epilogue<FUSED>(f, p, tbase + tl + ab * BN, m0, n0, smem + OFF_MISC + 256, q4, lane);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_ACCE + ab]);
                continue;
            }
            const int row = m0 + 32 * q4 + lane;
#pragma unroll 1
            for (int j = 0; j < BN / 32; ++j) {
                float v[32];
                tmem_ld32(tbase + tl + ab * BN + 32 * j, v);
                tmem_ld_wait();
                const int c0 = n0 + 32 * j;
                if (row >= p.M || c0 >= p.N) continue;
                // segment of the chunk's first column; a chunk inside one segment is stored as 4 x 16 bytes
                int sg = 0;
#pragma unroll
                for (int i = 1; i < 4; ++i)
                    if (i < p.nseg && c0 >= p.seg[i].col0) sg = i;
                const int seg_end = (sg + 1 < p.nseg) ? p.seg[sg + 1].col0 : p.N;
                if (c0 + 32 <= seg_end) {
                    uint16_t* dst = p.seg[sg].dst + (size_t)row * p.seg[sg].ld + (c0 - p.seg[sg].col0);
                    if ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            uint4 pk;
                            pk.x = pack_bf16x2(v[8 * e + 0], v[8 * e + 1]);
                            pk.y = pack_bf16x2(v[8 * e + 2], v[8 * e + 3]);
                            pk.z = pack_bf16x2(v[8 * e + 4], v[8 * e + 5]);
                            pk.w = pack_bf16x2(v[8 * e + 6], v[8 * e + 7]);
                            reinterpret_cast<uint4*>(dst)[e] = pk;
                        }
                        continue;
                    }
                }
                // ragged: element by element (segment boundaries, the last columns, unaligned rows)
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int c = c0 + e;
                    if (c < p.N) {
                        int s2 = 0;
#pragma unroll
                        for (int i = 1; i < 4; ++i)
                            if (i < p.nseg && c >= p.seg[i].col0) s2 = i;
                        p.seg[s2].dst[(size_t)row * p.seg[s2].ld + (c - p.seg[s2].col0)] = float_to_bf16_bits(v[e]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_ACCE + ab]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, TMEM_COLS);
}

}  // namespace gdn
