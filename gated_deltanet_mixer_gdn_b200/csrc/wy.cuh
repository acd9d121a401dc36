// Per-chunk WY representation of the gated delta rule, for every chunk at once.
//
// The recurrence (Qwen3.8 27B model card, "Gated DeltaNet" bullet), per value
// head with state S [128 v][128 k]:
//     S_t = exp(g_t) S_{t-1} + u_t k_t^T,   u_t = beta_t (v_t - exp(g_t) S_{t-1} k_t),
//     o_t = S_t q_t.
// Unrolled over a chunk of 64 tokens, with G the inclusive cumsum of g inside
// the chunk, A_ij = beta_i exp(G_i - G_j) (k_i . k_j) for j < i and
// T = (I + A)^-1, everything that does not involve the incoming state is
//     T1 = T diag(beta)                 (U~ = T1 V)
//     W  = T diag(beta e^G) K           (U = U~ - W S0^T)
//     M  = tril_incl(Q K^T) * E,  E_ij = exp(G_i - G_j)
// plus the decays e^{G_t}, e^{G_C - G_t} and e^{G_C} (the recurrence kernel
// scales Q and K by them: Qs = diag(e^G) Q, K' = diag(e^{G_C - G}) K).  None of it depends on the state,
// so this kernel computes it for all (chunk, value head) pairs in parallel and
// leaves a record per pair for the recurrence kernel (chunk.cuh).
//
// One task is (chunk, q/k head, up to three of its value heads).  Q K^T and
// K K^T are shared by the value heads of a q/k head, so one MMA1 serves the
// task; each value head then has its own warpgroup for the masked decays, the
// triangular inverse and its two products.  K K^T and Q K^T are formed from
// f16 hi/lo parts (hi.hi + hi.lo + lo.hi), which keeps the cancellation in
// q.k and k.k at f32 accuracy.
#pragma once

#include "common.cuh"
#include "prep.cuh"

namespace gdn {

struct WyParams {
    int Kh, Vh, total;
    SeqIndex seq;
    const int* chunk_base;  // [N+1] first chunk of each row (varlen), or nullptr for uniform rows
    int nchunks;            // chunks to process (all rows, or N * win for a window)
    int c0, win;            // uniform rows only: the chunk window [c0, c0 + win) of every row (win 0: all)
    const float* Gs;        // f32 [Vh][total] log-decay
    const float* Bs;        // f32 [Vh][total] write rate
    uint8_t* rec;           // records [nchunks][Vh] of wy::REC_BYTES
    int rec_chunks;         // chunks the record array holds (the index checks of the debug build)
};

namespace wy {
constexpr int C = 64;
constexpr int kHeads = 3;                 // value heads per task, one warpgroup each
constexpr int kThreads = 128 * kHeads;
constexpr int LDA = 68;                   // f32 row stride of A / T
// record of one (chunk, value head); the f16 tiles are stored as the byte
// image of a 128-byte-swizzled shared-memory tile (row r, 16-byte chunk c at
// r * 128 + ((c ^ (r & 7)) << 4)), so the reader moves them with plain bulk copies
constexpr uint32_t REC_T1 = 0;            // T diag(beta)            f16 [64 t][64 j]
constexpr uint32_t REC_MW = 8192;         // -W f16 [64 t][64 k] x 2 blocks (k 0-63, then 64-127)
constexpr uint32_t REC_M = 24576;         // tril_incl(Q K^T) * E    f16 [64 t][64 j]
constexpr uint32_t REC_DEC = 32768;       // f32 e^{G_C - G_t} [64], e^{G_t} [64], e^{G_C} (+ 12 bytes)
constexpr uint32_t REC_DEC_BYTES = 528;
constexpr uint32_t REC_BYTES = REC_DEC + REC_DEC_BYTES;
// shared memory (bytes from a 1024-aligned base)
// two input buffers (b = 0, 1 at b * IN_STRIDE), filled two tasks ahead
constexpr uint32_t IN_STRIDE = 65536;
constexpr uint32_t OFF_KQ = 0;            // [K t0-63 | Q t0-63] x k 0-63, then x k 64-127: f16 hi parts
constexpr uint32_t OFF_LO = 32768;        // same layout, lo parts
constexpr uint32_t OFF_T2 = 2 * IN_STRIDE;  // T diag(beta e^G) f16 [64][64], 8 KB per warpgroup
constexpr uint32_t OFF_WG = OFF_T2 + kHeads * 8192;  // per warpgroup: A / T f32 [64][LDA] and the solve scratch
constexpr uint32_t WG_BYTES = 64 * LDA * 4 + 32 * 36 * 4;
constexpr uint32_t OFF_MISC = OFF_WG + kHeads * WG_BYTES;
constexpr uint32_t MISC_BYTES = 4096;
constexpr uint32_t SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;
// misc: 0 barriers, 128 TMEM slot, 256 + 1024 * wg: G[64], e^G[64], beta[64], column decays[64]
constexpr uint32_t T_KQ = 0;              // [K;Q] K^T, 64 columns, of even tasks; W^T of warpgroup w at 64 (w + 1)
constexpr uint32_t T_KQ1 = 256;           // [K;Q] K^T of odd tasks (issued during the task before)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IN_BYTES = 8 * 8192;
constexpr uint32_t ID_KK = idesc_f16_f32(128, 64, false, false, false);
constexpr uint32_t ID_AMN = idesc_f16_f32(128, 64, true, false, false);
constexpr int B_IN = 0, B_MMA1 = 2, B_FREE = 4, B_W = 6;  // B_IN, B_MMA1, B_FREE + buffer; B_W + warpgroup
constexpr int kBars = B_W + kHeads;
}  // namespace wy

// ---- warp-level TF32 tensor-core products for the triangular solve.
// x = hi + lo with hi = x truncated to the 19 bits a tf32 operand carries (a
// bit mask on the integer pipe) and lo = x - hi (exact in f32; the tensor core
// keeps its top 19 bits); hi*hi + hi*lo + lo*hi recovers the product to about
// 2^-21 relative (the lo*lo term and lo's own truncation are below that).
__device__ __forceinline__ uint32_t tf32_hi(float x) { return __float_as_uint(x) & 0xffffe000u; }

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// acc[nt] (a 16 x 8 tile each) += A[16 x 8*KT] * B[8*KT x 8*NT]; A, B f32 in
// shared memory (row-major, strides lda / ldb); D fragment layout of m16n8.
template <int NT, int KT>
__device__ __forceinline__ void warp_gemm_tf32x3(float (&acc)[NT][4], const float* A, int lda, const float* B, int ldb,
                                                 int lane) {
    const int g = lane >> 2, t = lane & 3;
    float cor[NT][4] = {};  // hi*lo + lo*hi, kept apart so the MMA chains are independent
#pragma unroll
    for (int kt = 0; kt < KT; ++kt) {
        const float af[4] = {A[g * lda + kt * 8 + t], A[(g + 8) * lda + kt * 8 + t], A[g * lda + kt * 8 + t + 4],
                             A[(g + 8) * lda + kt * 8 + t + 4]};
        uint32_t ah[4], al[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            ah[i] = tf32_hi(af[i]);
            al[i] = __float_as_uint(af[i] - __uint_as_float(ah[i]));
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float bf[2] = {B[(kt * 8 + t) * ldb + nt * 8 + g], B[(kt * 8 + t + 4) * ldb + nt * 8 + g]};
            uint32_t bh[2], bl[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                bh[i] = tf32_hi(bf[i]);
                bl[i] = __float_as_uint(bf[i] - __uint_as_float(bh[i]));
            }
            mma_tf32(cor[nt], al, bh);
            mma_tf32(cor[nt], ah, bl);
            mma_tf32(acc[nt], ah, bh);
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] += cor[nt][i];
}

template <int NT>
__device__ __forceinline__ void warp_store_tile(float* D, int ldd, const float (&acc)[NT][4], float scale, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        D[g * ldd + nt * 8 + 2 * t] = scale * acc[nt][0];
        D[g * ldd + nt * 8 + 2 * t + 1] = scale * acc[nt][1];
        D[(g + 8) * ldd + nt * 8 + 2 * t] = scale * acc[nt][2];
        D[(g + 8) * ldd + nt * 8 + 2 * t + 1] = scale * acc[nt][3];
    }
}

// (I + A)^-1 of a unit lower-triangular 64 x 64 system, in place in sA (row
// stride LDA), by the 4 warps of one warpgroup (named barrier `bar`, 128
// threads; p = thread index in the warpgroup).  The four 16 x 16 diagonal
// blocks are inverted by forward substitution on the CUDA cores; the
// off-diagonal blocks follow from the block inverse [[Ta, 0], [Y, Tb]] with
// Y = -Tb * L_ba * Ta, first for the 16-blocks (1,0) and (3,2), then for the
// 32-block (1,0), on the tensor cores (f32-accurate TF32 products).
// sP: 32 x 36 f32 of scratch.
__device__ __forceinline__ void wy_tsolve(float* sA, float* sP, int p, uint32_t bar) {
    using wy::LDA;
    const int warp = p >> 5, lane = p & 31;
    // diagonal blocks, right-looking: once x_m is final it updates every later
    // row, so the dependency chain is 16 FMAs long
    float x[16];
    const int b = p >> 4, c = p & 15;
    if (p < 64) {
        const float* Ab = sA + (16 * b) * LDA + 16 * b;
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == c) ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m)
#pragma unroll
            for (int r = m + 1; r < 16; ++r) x[r] = fmaf(-Ab[r * LDA + m], x[m], x[r]);
    }
    named_barrier_sync(bar, 128);
    if (p < 64) {
        float* Ab = sA + (16 * b) * LDA + 16 * b;
#pragma unroll
        for (int r = 0; r < 16; ++r) Ab[r * LDA + c] = x[r];
    }
    named_barrier_sync(bar, 128);
    // 16-block merges (1,0) and (3,2): one 16 x 8 column tile per warp
    {
        const int bb = 2 * (warp >> 1), nt = warp & 1;
        float* X = sP + (warp >> 1) * 16 * 20;  // 16 x 16 scratch per merge, stride 20
        float acc[1][4] = {};
        warp_gemm_tf32x3<1, 2>(acc, sA + (16 * (bb + 1)) * LDA + 16 * bb, LDA, sA + (16 * bb) * LDA + 16 * bb + 8 * nt,
                               LDA, lane);
        warp_store_tile<1>(X + 8 * nt, 20, acc, 1.f, lane);
    }
    named_barrier_sync(bar, 128);
    {
        const int bb = 2 * (warp >> 1), nt = warp & 1;
        const float* X = sP + (warp >> 1) * 16 * 20;
        float acc[1][4] = {};
        warp_gemm_tf32x3<1, 2>(acc, sA + (16 * (bb + 1)) * LDA + 16 * (bb + 1), LDA, X + 8 * nt, 20, lane);
        warp_store_tile<1>(sA + (16 * (bb + 1)) * LDA + 16 * bb + 8 * nt, LDA, acc, -1.f, lane);
    }
    named_barrier_sync(bar, 128);
    // 32-block merge: one 16 x 16 quadrant per warp
    const int mi = warp >> 1, ni = warp & 1;
    {
        float acc[2][4] = {};
        warp_gemm_tf32x3<2, 4>(acc, sA + (32 + 16 * mi) * LDA, LDA, sA + 16 * ni, LDA, lane);
        warp_store_tile<2>(sP + (16 * mi) * 36 + 16 * ni, 36, acc, 1.f, lane);
    }
    named_barrier_sync(bar, 128);  // X complete; every read of L_ba is done
    {
        float acc[2][4] = {};
        warp_gemm_tf32x3<2, 4>(acc, sA + (32 + 16 * mi) * LDA + 32, LDA, sP + 16 * ni, 36, lane);
        warp_store_tile<2>(sA + (32 + 16 * mi) * LDA + 16 * ni, LDA, acc, -1.f, lane);
    }
    named_barrier_sync(bar, 128);
}

// Row of the chunk-wide cumulative decay: G_t = sum_{s <= t} g_s over the
// first 64 threads p of a group (two warps), through `sG` and barrier `bar`.
// Tokens past the end of the row carry g = 0.
__device__ __forceinline__ float chunk_cumsum(float g, float* sG, int p, int lane, uint32_t bar, uint32_t nthreads) {
    float x = g;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (p < 64) sG[p] = x;
    named_barrier_sync(bar, nthreads);
    const float Gi = (p < 64) ? x + ((p >= 32) ? sG[31] : 0.f) : 0.f;
    named_barrier_sync(bar, nthreads);
    if (p < 64) sG[p] = Gi;
    named_barrier_sync(bar, nthreads);
    return Gi;
}

// cb[n] = number of 64-token chunks in rows 0..n-1 (cb[0] = 0, cb[N] = all),
// from cu_seqlens; one block of 1024 threads walks the rows in tiles.
// ord[0..N): the rows by length, longest first (ties: lower index first), by a bitonic
// sort in shared memory when N <= kOrderMax; otherwise the identity.  The recurrence
// launches its rows in this order, so the longest rows are not left for the last wave.
constexpr int kOrderMax = 2048;
__global__ void __launch_bounds__(1024) gdn_chunk_base_kernel(const int* cu, int N, int* cb, int* ord) {
    __shared__ int s_warp[32];
    __shared__ int s_carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        s_carry = 0;
        cb[0] = 0;
    }
    __syncthreads();
    for (int base = 0; base < N; base += 1024) {
        const int i = base + tid;
        const int v = (i < N) ? (__ldg(cu + i + 1) - __ldg(cu + i) + wy::C - 1) / wy::C : 0;
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) s_warp[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int w = s_warp[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            s_warp[lane] = w;  // inclusive over warps
        }
        __syncthreads();
        const int carry = s_carry;
        const int incl = carry + x + (warp > 0 ? s_warp[warp - 1] : 0);
        if (i < N) cb[i + 1] = incl;
        __syncthreads();
        if (tid == 1023) s_carry = incl;
        __syncthreads();
    }
    if (ord == nullptr) return;
    if (N > kOrderMax) {
        for (int i = tid; i < N; i += 1024) ord[i] = i;
        return;
    }
    __shared__ unsigned long long s_key[kOrderMax];
    int P = 2;
    while (P < N) P <<= 1;
    for (int i = tid; i < P; i += 1024) {  // key: (INT_MAX - length, index); padding sorts last
        const int len = i < N ? __ldg(cu + i + 1) - __ldg(cu + i) : 0;
        s_key[i] = i < N ? ((unsigned long long)(0x7fffffff - len) << 32) | (unsigned)i : ~0ull;
    }
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < P; i += 1024) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const unsigned long long x = s_key[i], y = s_key[ixj];
                    if ((x > y) == ((i & k) == 0)) {
                        s_key[i] = y;
                        s_key[ixj] = x;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int i = tid; i < N; i += 1024) ord[i] = (int)(s_key[i] & 0xffffffffu);
}

// Row n and chunk index c of global chunk g.
__device__ __forceinline__ void chunk_row(const WyParams& p, int g, int& n, int& c) {
    if (p.chunk_base == nullptr) {
        const int per = (p.seq.uniform_T + wy::C - 1) / wy::C;
        n = g / per;
        c = g - n * per;
        return;
    }
    int lo = 0, hi = p.seq.N;  // chunk_base[lo] <= g < chunk_base[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(p.chunk_base + mid) <= g) lo = mid;
        else hi = mid;
    }
    n = lo;
    c = g - __ldg(p.chunk_base + n);
}

__global__ void __launch_bounds__(wy::kThreads, 1)
    gdn_wy_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmKl, const __grid_constant__ CUtensorMap tmQl,
                  const WyParams p) {
    using namespace wy;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int wg = warp >> 2;              // warpgroup = value head slot
    const int wt = tid & 127;              // thread in the warpgroup
    const int row = 32 * (warp & 3) + lane;  // TMEM lane of this thread
    const uint32_t wbar = 1 + wg;          // named barrier of the warpgroup

    uint8_t* misc = smem + OFF_MISC;
    uint64_t* bars = reinterpret_cast<uint64_t*>(misc);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(misc + 128);
    float* sG = reinterpret_cast<float*>(misc + 256 + 1024 * wg);
    float* seG = sG + 64;
    float* sbeta = sG + 128;
    float* scol = sG + 192;  // e^{G_r - G_j}, r the last token of j's 16-token block
    float* sA = reinterpret_cast<float*>(smem + OFF_WG + wg * WG_BYTES);
    float* sP = sA + 64 * LDA;
    uint8_t* sT2 = smem + OFF_T2 + 8192 * wg;

    const int ratio = p.Vh / p.Kh;
    const int nsub = (ratio + kHeads - 1) / kHeads;
    const int ntasks = p.nchunks * p.Kh * nsub;

    if (tid == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars[B_IN + b], 1);
            mbar_init(&bars[B_FREE + b], kHeads);
        }
        mbar_init(&bars[B_MMA1], 1);
        mbar_init(&bars[B_MMA1 + 1], 1);
        for (int w = 0; w < kHeads; ++w) mbar_init(&bars[B_W + w], 1);
        fence_barrier_init();
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmKl);
        prefetch_tensormap(&tmQl);
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem;
    const uint32_t tlane = tbase + (static_cast<uint32_t>(32 * (warp & 3)) << 16);

    // task -> (global chunk, q/k head, value-head subset)
    auto task_coords = [&](int task, int& g, int& kap, int& sub) {
        sub = task % nsub;
        const int r = task / nsub;
        kap = r % p.Kh;
        g = r / p.Kh;
        if (p.win > 0) {  // window chunk -> chunk of the row
            const int per = (p.seq.uniform_T + C - 1) / C;
            g = (g / p.win) * per + p.c0 + g % p.win;
        }
    };
    auto issue_loads = [&](int task, int b) {
        int g, kap, sub, n, c;
        task_coords(task, g, kap, sub);
        chunk_row(p, g, n, c);
        int start, len;
        p.seq.bounds(n, start, len);
        const int y = start + c * C;
        uint8_t* in = smem + b * IN_STRIDE;
        uint64_t* full = &bars[B_IN + b];
        mbar_arrive_expect_tx(full, IN_BYTES);
        tma_load_2d(in + OFF_KQ, &tmK, kap * 128, y, full);
        tma_load_2d(in + OFF_KQ + 16384, &tmK, kap * 128 + 64, y, full);
        tma_load_2d(in + OFF_KQ + 8192, &tmQ, kap * 128, y, full);
        tma_load_2d(in + OFF_KQ + 24576, &tmQ, kap * 128 + 64, y, full);
        tma_load_2d(in + OFF_LO, &tmKl, kap * 128, y, full);
        tma_load_2d(in + OFF_LO + 16384, &tmKl, kap * 128 + 64, y, full);
        tma_load_2d(in + OFF_LO + 8192, &tmQl, kap * 128, y, full);
        tma_load_2d(in + OFF_LO + 24576, &tmQl, kap * 128 + 64, y, full);
    };
    if (tid == 0) {  // the first two tasks of this CTA
        if ((int)blockIdx.x < ntasks) issue_loads(blockIdx.x, 0);
        if ((int)(blockIdx.x + gridDim.x) < ntasks) issue_loads(blockIdx.x + gridDim.x, 1);
    }

    bool broken = false;
    auto wait = [&](int slot, uint32_t parity) {
        if (!broken && !mbar_wait(&bars[slot], parity)) {
            broken = true;
            record_error(kErrTimeoutTma);
        }
        __syncwarp();
    };
    // the same for a single thread
    auto wait1 = [&](int slot, uint32_t parity) {
        if (!broken && !mbar_wait(&bars[slot], parity)) {
            broken = true;
            record_error(kErrTimeoutTma);
        }
    };

    // gate inputs of a task (value head slot of this warpgroup, token wt), loaded a task ahead
    auto load_gates = [&](int task, float& gv, float& bv) {
        gv = 0.f;
        bv = 0.f;
        if (task >= ntasks || wt >= C) return;
        int g, kap, sub, n, c;
        task_coords(task, g, kap, sub);
        chunk_row(p, g, n, c);
        const int hslot = sub * kHeads + wg;
        if (hslot >= ratio) return;
        int start, len;
        p.seq.bounds(n, start, len);
        if (wt < min(C, len - c * C) && GDN_CHECK(start + c * C + wt < p.total && kap * ratio + hslot < p.Vh)) {
            const size_t off = (size_t)(kap * ratio + hslot) * p.total + start + c * C + wt;
            gv = __ldg(p.Gs + off);
            bv = __ldg(p.Bs + off);
        }
    };
    float gv_next, bv_next;
    load_gates(blockIdx.x, gv_next, bv_next);

    // MMA1 of the task in input buffer b: [K;Q] K^T from hi/lo f16 parts into accumulator b
    // (one thread).  The task's own MMA1 was issued during the task before it, so the
    // tensor core runs it while that task solves its triangular system.
    auto issue_mma1 = [&](int b, uint32_t parity) {
        wait1(B_IN + b, parity);
        tc_fence_after();
        const uint32_t aKQ = sbase + b * IN_STRIDE + OFF_KQ, aLO = sbase + b * IN_STRIDE + OFF_LO;
        const uint32_t d = tbase + (b ? T_KQ1 : T_KQ);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
            mma_f16(d, sw128_desc(aKQ + off, 16, 1024), sw128_desc(aKQ + off, 16, 1024), ID_KK, s > 0);
        }
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
            mma_f16(d, sw128_desc(aKQ + off, 16, 1024), sw128_desc(aLO + off, 16, 1024), ID_KK, 1);
        }
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
            mma_f16(d, sw128_desc(aLO + off, 16, 1024), sw128_desc(aKQ + off, 16, 1024), ID_KK, 1);
        }
        mma_commit(&bars[B_MMA1 + b]);
    };
    if (tid == 0 && (int)blockIdx.x < ntasks) issue_mma1(0, 0);
    __syncwarp();

    uint32_t it = 0;
    for (int task = blockIdx.x; task < ntasks; task += gridDim.x, ++it) {
        const uint32_t ph = it & 1;          // barriers used once per task
        const int buf = it & 1;              // input buffer of this task
        const uint32_t pb = (it >> 1) & 1;   // barriers of that buffer: used every other task
        const uint32_t in_base = sbase + buf * IN_STRIDE;
        int g, kap, sub, n, c;
        task_coords(task, g, kap, sub);
        chunk_row(p, g, n, c);
        int start, len;
        p.seq.bounds(n, start, len);
        const int tok0 = start + c * C;
        const int nv = min(C, len - c * C);
        const int hslot = sub * kHeads + wg;
        const bool active = hslot < ratio;
        const int h = kap * ratio + hslot;
        // (debug build: a record index out of range is recorded and the task writes record 0)
        const bool rec_ok = !active || GDN_CHECK(g >= 0 && g < p.rec_chunks && h < p.Vh);
        uint8_t* rec = p.rec + (rec_ok ? ((size_t)g * p.Vh + h) * REC_BYTES : 0);

        const float gv = gv_next, bv = bv_next;
        load_gates(task + gridDim.x, gv_next, bv_next);
        (void)tok0;
        (void)nv;

        // ---- gates: G, e^G, beta, the column decays; the decay part of the record
        if (active) {
            const float Gi = chunk_cumsum(gv, sG, wt, lane, wbar, 128);
            if (wt < 64) {
                const float e = expf(Gi);
                seG[wt] = e;
                sbeta[wt] = bv;
                scol[wt] = expf(sG[wt | 15] - Gi);
                float* dec = reinterpret_cast<float*>(rec + REC_DEC);
                dec[wt] = expf(sG[63] - Gi);
                dec[64 + wt] = e;
                if (wt == 63) dec[128] = e;
            }
            named_barrier_sync(wbar, 128);
        }
        wait(B_MMA1 + buf, pb);
        tc_fence_after();

        if (!active) {
            // nothing to do for this slot; the input buffer is not read by it
            if (wt == 0) mbar_arrive(&bars[B_FREE + buf]);
            __syncwarp();
        } else {
            // ---- A (rows of K K^T) and M (rows of Q K^T), masked before the exp
            {
                const bool is_a = row < 64;
                const int i = is_a ? row : row - 64;
                const int last = is_a ? i - 1 : i;  // last unmasked column
                const int I = i >> 4;               // 16-token block of the row
                const float Gr = sG[i], scale = is_a ? sbeta[i] : 1.f;
                // e^{G_i - G_j} = e^{G_i - G_r} e^{G_r - G_j} for j in an earlier block (r its last
                // token, both factors <= 1); direct exponentials inside the row's own block
                // the first half of the row is read from TMEM while the exponentials are formed
                const uint32_t tkq = tlane + (buf ? T_KQ1 : T_KQ);
                float v[32];
                tmem_ld32(tkq, v);
                float rowf[3], diag[16];
#pragma unroll
                for (int J = 0; J < 3; ++J) rowf[J] = (J < I) ? scale * __expf(Gr - sG[16 * J + 15]) : 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const int j = 16 * I + m;
                    diag[m] = (j <= last) ? scale * __expf(Gr - sG[j]) : 0.f;
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    if (hh == 1) tmem_ld32(tkq + 32, v);
                    tmem_ld_wait();
                    float e[32];
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int j = 32 * hh + jj;
                        const int J = j >> 4;
                        const float f = (J < 3 && J < I) ? rowf[J < 3 ? J : 0] * scol[j] : 0.f;
                        e[jj] = ((J == I) ? diag[j & 15] : f) * v[jj];
                    }
                    if (is_a) {
                        float4* dst = reinterpret_cast<float4*>(sA + i * LDA + 32 * hh);
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4)
                            dst[j4] = make_float4(e[4 * j4], e[4 * j4 + 1], e[4 * j4 + 2], e[4 * j4 + 3]);
                    } else {
                        store_row_f16_sw128(rec + REC_M, i, 4 * hh, e, 1.f);
                    }
                }
            }
            named_barrier_sync(wbar, 128);
            tc_fence_before();
            // the next task's MMA1 (its accumulator was last read two tasks ago, and every
            // warpgroup has passed that task's MMA3)
            if (tid == 0 && task + (int)gridDim.x < ntasks) issue_mma1(buf ^ 1, ((it + 1) >> 1) & 1);
            __syncwarp();

            // ---- T = (I + A)^-1; T diag(beta) to the record, T diag(beta e^G) to shared memory
            // (the warpgroup's own 8 KB, read by its MMA3)
            wy_tsolve(sA, sP, wt, wbar);
            {
                const int t = wt >> 1, hh = wt & 1;
                const float* Tr = sA + t * LDA + 32 * hh;
                float t1[32], t2[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int tp = 32 * hh + e;
                    t1[e] = Tr[e] * sbeta[tp];
                    t2[e] = t1[e] * seG[tp];
                }
                store_row_f16_sw128(sT2, t, 4 * hh, t2, 1.f);
                store_row_f16_sw128(rec + REC_T1, t, 4 * hh, t1, 1.f);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_barrier_sync(wbar, 128);

            // ---- MMA3: W^T = K^T (T diag(beta e^G))^T
            if (wt == 0) {
                tc_fence_after();
                const uint32_t tW = tbase + 64 * (wg + 1);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_f16(tW, sw128_desc(in_base + OFF_KQ + s * 2048, 16384, 1024),
                            sw128_desc(smem_u32(sT2) + s * 32, 16, 1024), ID_AMN, s > 0);
                mma_commit(&bars[B_W + wg]);
                mma_commit(&bars[B_FREE + buf]);
            }
            __syncwarp();
        }

        // ---- -W to the record: TMEM lane k holds column k of W (64 tokens)
        if (active) {
            wait(B_W + wg, ph);
            tc_fence_after();
            // Lanes k (even) and k + 1 swap halves of their packed token pairs, so that the even
            // lane stores columns k, k + 1 of token t and the odd lane those of token t + 1.
            const uint32_t odd = row & 1;
            uint8_t* dst = rec + REC_MW + (row >> 6) * 8192 + (row & 6) * 2;
            const uint32_t kc = (row & 63) >> 3;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float v[32];
                tmem_ld32(tlane + 64 * (wg + 1) + 32 * hh, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; j += 2) {  // tokens 32 hh + j, + 1 of column k = row
                    const uint32_t pr = pack_half2(-v[j], -v[j + 1]);
                    const uint32_t q = __shfl_xor_sync(0xffffffffu, pr, 1);
                    const uint32_t word = odd ? ((q >> 16) | (pr & 0xffff0000u)) : ((pr & 0xffffu) | (q << 16));
                    *reinterpret_cast<uint32_t*>(dst + sw128_chunk(32 * hh + j + odd, kc)) = word;
                }
            }
            tc_fence_before();
        }

        // ---- once every slot is done with this buffer, fill it with the task after next
        // (after this warpgroup's own record, so its thread 0 does not wait for the others first)
        if (tid == 0) {
            wait1(B_FREE + buf, pb);
            if (task + 2 * (int)gridDim.x < ntasks) issue_loads(task + 2 * gridDim.x, buf);
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, TMEM_COLS);
}

}  // namespace gdn
