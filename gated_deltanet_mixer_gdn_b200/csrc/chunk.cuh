// Chunked prefill of the gated delta rule on 5th-generation tensor cores.
//
// The recurrence (Qwen3.8 27B model card, "Gated DeltaNet" bullet), per value
// head with state S [128 v][128 k]:
//     S_t = exp(g_t) S_{t-1} + u_t k_t^T,   u_t = beta_t (v_t - exp(g_t) S_{t-1} k_t),
//     o_t = S_t q_t.
// In chunks of 64 tokens with G = inclusive cumsum of g inside the chunk,
// A_ij = beta_i exp(G_i - G_j) (k_i . k_j) for j < i and T = (I + A)^-1:
//     U   = T diag(beta) V - T diag(beta e^G) K S0^T   ( = U~ - W S0^T )
//     O   = diag(e^G) Q S0^T + (tril_incl(Q K^T) * E) U,   E_ij = exp(G_i - G_j)
//     S_C = e^{G_C} S0 + U^T diag(e^{G_C - G}) K.
// (Obtained by unrolling the recurrence inside a chunk; every ratio of decays
// is formed as exp of a difference over j <= i, so nothing overflows.)
//
// One CTA owns one (row, value head) and walks its chunks in order.  All seven
// contractions run as tcgen05.mma (f16 operands in 128B-swizzled shared
// memory, f32 accumulators in TMEM), arranged so that M = 128 every time:
//   MMA1  KQ   [128 x 64]  = [K;Q] K^T                (A K-major, B K-major)
//   MMA2  U~^T [128v x 64] = V^T (T diag beta)^T       (A = V tile read MN-major)
//   MMA3  W^T  [128k x 64] = K^T (T diag(beta e^G))^T  (A = K tile read MN-major)
//   MMA4  U^T  += -S0 W^T                             (negated A, B = W^T MN-major)
//   MMA5  Oi^T [128v x 64] = S0 Q^T                    (e^G applied in the epilogue)
//   MMA6  dS   [128v x128k]= (U^T diag e^{G_C-G}) K    (B = K tile read MN-major)
//   MMA7  Oa^T [128v x 64] = U^T (tril(QK^T)*E)^T
// The unit lower-triangular inverse T is formed on the CUDA cores (blocked
// 16 x 16 forward substitution in f32).  The state lives in registers in
// f32 (thread = one v row, one half of k) and is re-staged as f16 in shared
// memory for the next chunk.  The gated RMSNorm is fused into the epilogue
// and the 64 x 128 bf16 output tile leaves with coalesced 16-byte stores.
//
// Inputs come from the load-stage kernel (conv, L2 norm, gates) as f16 tiles
// fetched with TMA: K and Q of the q/k head (double-buffered) with their f16
// residuals, V of the value head, and the z tile for the gate of the norm.
// MMA1 uses the residuals (hi.hi + hi.lo + lo.hi): the dot products of nearly
// orthogonal q and k cancel, and one f16 rounding of q and k then dominates
// the error of the normalised outputs.
#pragma once

#include "common.cuh"
#include "prep.cuh"

namespace gdn {

struct ChunkParams {
    int Kh, Vh, total;
    SeqIndex seq;
    const float* Gs;          // f32 [Vh][total] log-decay
    const float* Bs;          // f32 [Vh][total] write rate
    const float* init_state;  // f32 [N][Vh][128][128] or nullptr
    float* final_state;       // f32 [N][Vh][128][128] or nullptr (may alias init_state)
    const float* norm_w;      // f32 [128]
    uint16_t* out;            // bf16 [total][Vh*128]
};

namespace chunk {
constexpr int C = 64;              // tokens per chunk
constexpr int kThreads = 256;
constexpr int LDA = 68;            // f32 row stride of the A / T matrix (conflict-free float4 rows)
// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ0 = 0;        // [K rows 0-63 | Q rows 64-127] x k 0-63, then x k 64-127 (f16 hi parts)
constexpr uint32_t OFF_KQ1 = 32768;    // second buffer
constexpr uint32_t OFF_LO = 65536;     // same layout, f16 residuals (lo parts); A / T f32 once MMA1 is done
constexpr uint32_t OFF_V = 98304;      // V [64 t][64 v] x 2 blocks
constexpr uint32_t OFF_WT = 114688;    // W^T f16 [128 k][64 t]; z / y bf16 [64][128] once MMA4 is done
constexpr uint32_t OFF_UT = 131072;    // U^T f16 [128 v][64 t]; T-solve scratch before that
constexpr uint32_t OFF_UTS = 147456;   // U^T diag(e^{G_C-G}) f16
constexpr uint32_t OFF_S = 163840;     // S0 f16 [128 v][64 k] x 2 blocks
constexpr uint32_t OFF_T1 = 196608;    // T diag(beta) f16 [64][64]
constexpr uint32_t OFF_T2 = 204800;    // T diag(beta e^G) f16 [64][64]
constexpr uint32_t OFF_M = 212992;     // tril(Q K^T) * E f16 [64][64]
constexpr uint32_t OFF_A = OFF_LO;     // A, then T, f32 [64][LDA]
constexpr uint32_t OFF_Z = OFF_WT;
constexpr uint32_t OFF_MISC = 221184;
constexpr uint32_t MISC_BYTES = 3072;
constexpr uint32_t SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;  // + alignment slack
static_assert(64 * LDA * 4 <= 32768, "A/T must fit in the residual tile");
// TMEM columns (f32, 128 lanes)
constexpr uint32_t T_KQ = 0, T_UT = 64, T_WT = 128, T_OI = 192, T_OA = 256, T_S = 320;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t KQV_BYTES = 6 * 8192;
constexpr uint32_t LO_BYTES = 4 * 8192;
constexpr uint32_t Z_BYTES = 64 * 128 * 2;
constexpr uint32_t ID_KK = idesc_f16_f32(128, 64, false, false, false);
constexpr uint32_t ID_AMN = idesc_f16_f32(128, 64, true, false, false);
constexpr uint32_t ID_NEG_BMN = idesc_f16_f32(128, 64, false, true, true);
constexpr uint32_t ID_DS = idesc_f16_f32(128, 128, false, true, false);
}  // namespace chunk

// ---- warp-level TF32 tensor-core products for the triangular solve.
// x = hi + lo with hi, lo representable in tf32; hi*hi + hi*lo + lo*hi
// recovers an f32-accurate product (the lo*lo term is below f32 rounding).
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

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
#pragma unroll
    for (int kt = 0; kt < KT; ++kt) {
        const float af[4] = {A[g * lda + kt * 8 + t], A[(g + 8) * lda + kt * 8 + t], A[g * lda + kt * 8 + t + 4],
                             A[(g + 8) * lda + kt * 8 + t + 4]};
        uint32_t ah[4], al[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            ah[i] = to_tf32(af[i]);
            al[i] = to_tf32(af[i] - __uint_as_float(ah[i]));
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float bf[2] = {B[(kt * 8 + t) * ldb + nt * 8 + g], B[(kt * 8 + t + 4) * ldb + nt * 8 + g]};
            uint32_t bh[2], bl[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                bh[i] = to_tf32(bf[i]);
                bl[i] = to_tf32(bf[i] - __uint_as_float(bh[i]));
            }
            mma_tf32(acc[nt], al, bh);
            mma_tf32(acc[nt], ah, bl);
            mma_tf32(acc[nt], ah, bh);
        }
    }
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
// stride LDA).  The four 16 x 16 diagonal blocks are inverted by forward
// substitution on the CUDA cores; the off-diagonal blocks follow from the
// block inverse [[Ta, 0], [Y, Tb]] with Y = -Tb * L_ba * Ta, first for the
// 16-blocks (1,0) and (3,2), then for the 32-block (1,0), on the tensor cores
// (f32-accurate TF32 products).  sP: 4 KiB of f32 scratch.
__device__ __forceinline__ void chunk_tsolve(float* sA, float* sP, int tid) {
    using namespace chunk;
    const int warp = tid >> 5, lane = tid & 31;
    float x[16];
    const int b = tid >> 4, c = tid & 15;
    if (tid < 64) {
        const float* Ab = sA + (16 * b) * LDA + 16 * b;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float s = 0.f;
#pragma unroll
            for (int m = 0; m < r; ++m) s = fmaf(Ab[r * LDA + m], x[m], s);
            x[r] = (r == c) ? 1.f : ((r < c) ? 0.f : -s);
        }
    }
    __syncthreads();
    if (tid < 64) {
        float* Ab = sA + (16 * b) * LDA + 16 * b;
#pragma unroll
        for (int r = 0; r < 16; ++r) Ab[r * LDA + c] = x[r];
    }
    __syncthreads();
    // 16-block merges: warp 0 -> block (1,0), warp 1 -> block (3,2)
    if (warp < 2) {
        const int bb = 2 * warp;                 // upper-left block index of the pair
        float* X = sP + warp * 16 * 20;          // 16 x 16 scratch, stride 20
        float acc[2][4] = {};
        warp_gemm_tf32x3<2, 2>(acc, sA + (16 * (bb + 1)) * LDA + 16 * bb, LDA, sA + (16 * bb) * LDA + 16 * bb, LDA,
                               lane);
        warp_store_tile<2>(X, 20, acc, 1.f, lane);
        __syncwarp();
        float acc2[2][4] = {};
        warp_gemm_tf32x3<2, 2>(acc2, sA + (16 * (bb + 1)) * LDA + 16 * (bb + 1), LDA, X, 20, lane);
        warp_store_tile<2>(sA + (16 * (bb + 1)) * LDA + 16 * bb, LDA, acc2, -1.f, lane);
    }
    __syncthreads();
    // 32-block merge: warps 0-3, one 16 x 16 quadrant each
    if (warp < 4) {
        const int mi = warp >> 1, ni = warp & 1;
        float* X = sP;  // 32 x 32 scratch, stride 36
        float acc[2][4] = {};
        warp_gemm_tf32x3<2, 4>(acc, sA + (32 + 16 * mi) * LDA, LDA, sA + 16 * ni, LDA, lane);
        warp_store_tile<2>(X + (16 * mi) * 36 + 16 * ni, 36, acc, 1.f, lane);
        named_barrier_sync(2, 128);
        float acc2[2][4] = {};
        warp_gemm_tf32x3<2, 4>(acc2, sA + (32 + 16 * mi) * LDA + 32, LDA, X + 16 * ni, 36, lane);
        named_barrier_sync(2, 128);  // every quadrant of X is read before L_ba is overwritten
        warp_store_tile<2>(sA + (32 + 16 * mi) * LDA + 16 * ni, LDA, acc2, -1.f, lane);
    }
    __syncthreads();
}

// Lane l of the warp ends with sum over the 32 lanes of v[l] (31 shuffles).
__device__ __forceinline__ float warp_transpose_sum(float (&v)[32], int lane) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
            const float send = upper ? v[i] : v[i + off];
            const float keep = upper ? v[i + off] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    return v[0];
}

__device__ __forceinline__ void store_row_f16_sw128(uint8_t* tile, uint32_t row, uint32_t chunk0, const float* vals,
                                                    float scale_all) {
    // 32 values -> 4 chunks of 8 f16 starting at 16-byte chunk index chunk0
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint4 pk;
        pk.x = pack_half2(vals[8 * j + 0] * scale_all, vals[8 * j + 1] * scale_all);
        pk.y = pack_half2(vals[8 * j + 2] * scale_all, vals[8 * j + 3] * scale_all);
        pk.z = pack_half2(vals[8 * j + 4] * scale_all, vals[8 * j + 5] * scale_all);
        pk.w = pack_half2(vals[8 * j + 6] * scale_all, vals[8 * j + 7] * scale_all);
        *reinterpret_cast<uint4*>(tile + sw128_chunk(row, chunk0 + j)) = pk;
    }
}

#define CHUNK_WAIT(bar, parity, code)                  \
    {                                                  \
        const bool ok_ = mbar_wait((bar), (parity));   \
        if (__syncthreads_or(!ok_)) {                  \
            if (tid == 0) record_error(code);          \
            failed = true;                             \
            break;                                     \
        }                                              \
    }

__global__ void __launch_bounds__(chunk::kThreads, 1)
    gdn_chunk_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmKl, const __grid_constant__ CUtensorMap tmQl,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmZ,
                     const ChunkParams p) {
    using namespace chunk;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);

    const int h = blockIdx.x;
    const int n = blockIdx.y;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3;        // TMEM lane quarter of this warp
    const int hf = warp >> 2;       // column half handled by this warp
    const int row = 32 * q4 + lane; // TMEM lane = v row / k row / token row
    const int kap = h / (p.Vh / p.Kh);

    uint64_t* bar_kqv = reinterpret_cast<uint64_t*>(smem + OFF_MISC);
    uint64_t* bar_z = bar_kqv + 1;
    uint64_t* bar_mma = bar_kqv + 2;
    uint64_t* bar_lo = bar_kqv + 3;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + OFF_MISC + 32);
    float* s_G = reinterpret_cast<float*>(smem + OFF_MISC + 64);     // [64]
    float* s_eG = s_G + 64;                                            // [64]
    float* s_beta = s_G + 128;                                         // [64]
    float* s_red = reinterpret_cast<float*>(smem + OFF_MISC + 1024);  // [4][64]
    float* s_rstd = reinterpret_cast<float*>(smem + OFF_MISC + 2048); // [64]
    float* sA = reinterpret_cast<float*>(smem + OFF_A);
    float* sP = reinterpret_cast<float*>(smem + OFF_UT);

    int start, len;
    p.seq.bounds(n, start, len);
    const int nchunks = (len + C - 1) / C;

    if (tid == 0) {
        mbar_init(bar_kqv, 1);
        mbar_init(bar_z, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_lo, 1);
        fence_barrier_init();
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmKl);
        prefetch_tensormap(&tmQl);
        prefetch_tensormap(&tmV);
        prefetch_tensormap(&tmZ);
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem;
    const uint32_t tlane = tbase + (static_cast<uint32_t>(32 * q4) << 16);

    // Initial state: thread holds S[row][64*hf .. 64*hf+63] in f32.
    float S[64];
    {
        const float* src = p.init_state ? p.init_state + (((size_t)n * p.Vh + h) * 128 + row) * 128 + 64 * hf : nullptr;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            float4 v = src ? __ldg(reinterpret_cast<const float4*>(src) + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[4 * j] = v.x;
            S[4 * j + 1] = v.y;
            S[4 * j + 2] = v.z;
            S[4 * j + 3] = v.w;
        }
        uint8_t* sS = smem + OFF_S + 16384 * hf;
        store_row_f16_sw128(sS, row, 0, S, 1.f);
        store_row_f16_sw128(sS, row, 4, S + 32, 1.f);
    }
    fence_proxy_async_smem();
    if (tid == 0 && nchunks > 0) {
        mbar_arrive_expect_tx(bar_kqv, KQV_BYTES);
        tma_load_2d(smem + OFF_KQ0, &tmK, kap * 128, start, bar_kqv);
        tma_load_2d(smem + OFF_KQ0 + 16384, &tmK, kap * 128 + 64, start, bar_kqv);
        tma_load_2d(smem + OFF_KQ0 + 8192, &tmQ, kap * 128, start, bar_kqv);
        tma_load_2d(smem + OFF_KQ0 + 24576, &tmQ, kap * 128 + 64, start, bar_kqv);
        tma_load_2d(smem + OFF_V, &tmV, h * 128, start, bar_kqv);
        tma_load_2d(smem + OFF_V + 8192, &tmV, h * 128 + 64, start, bar_kqv);
        mbar_arrive_expect_tx(bar_lo, LO_BYTES);
        tma_load_2d(smem + OFF_LO, &tmKl, kap * 128, start, bar_lo);
        tma_load_2d(smem + OFF_LO + 16384, &tmKl, kap * 128 + 64, start, bar_lo);
        tma_load_2d(smem + OFF_LO + 8192, &tmQl, kap * 128, start, bar_lo);
        tma_load_2d(smem + OFF_LO + 24576, &tmQl, kap * 128 + 64, start, bar_lo);
    }
    __syncthreads();

    const float wn = 1.0f + __ldg(p.norm_w + row);  // (1 + w) of this thread's v channel
    bool failed = false;
    // gate inputs of the next chunk, loaded one chunk ahead (threads tid < 64)
    float g_next = 0.f, b_next = 0.f;
    if (tid < 64 && nchunks > 0 && tid < min(C, len)) {
        g_next = __ldg(p.Gs + (size_t)h * p.total + start + tid);
        b_next = __ldg(p.Bs + (size_t)h * p.total + start + tid);
    }
    uint32_t mma_phase = 0;

    for (int c = 0; c < nchunks; ++c) {
        const int tok0 = start + c * C;
        const int nv = min(C, len - c * C);
        const uint32_t kq_off = (c & 1) ? OFF_KQ1 : OFF_KQ0;
        const uint32_t aKQ = sbase + kq_off;

        // ---- gates of the chunk: G = inclusive cumsum of g, e^G, beta
        if (tid < 64) {
            const float g = g_next, bt = b_next;
            const int nv1 = min(C, len - (c + 1) * C);  // tokens of the next chunk (<= 0: none)
            g_next = (tid < nv1) ? __ldg(p.Gs + (size_t)h * p.total + tok0 + C + tid) : 0.f;
            b_next = (tid < nv1) ? __ldg(p.Bs + (size_t)h * p.total + tok0 + C + tid) : 0.f;
            float x = g;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            s_G[tid] = x;
            s_beta[tid] = bt;
        }
        CHUNK_WAIT(bar_kqv, c & 1, kErrTimeoutTma);  // includes a CTA barrier
        CHUNK_WAIT(bar_lo, c & 1, kErrTimeoutTma);
        if (tid < 64) {
            float G = s_G[tid];
            if (tid >= 32) G += s_G[31];
            s_G[tid] = G;
            s_eG[tid] = expf(G);
        }
        // ---- MMA1: [K;Q] K^T from hi/lo f16 parts: hi.hi + hi.lo + lo.hi
        if (tid == 0) {
            tc_fence_after();
            const uint32_t aLO = sbase + OFF_LO;
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                mma_f16(tbase + T_KQ, sw128_desc(aKQ + off, 16, 1024), sw128_desc(aKQ + off, 16, 1024), ID_KK,
                        s > 0);
            }
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                mma_f16(tbase + T_KQ, sw128_desc(aKQ + off, 16, 1024), sw128_desc(aLO + off, 16, 1024), ID_KK, 1);
            }
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                mma_f16(tbase + T_KQ, sw128_desc(aLO + off, 16, 1024), sw128_desc(aKQ + off, 16, 1024), ID_KK, 1);
            }
            mma_commit(bar_mma);
        }
        CHUNK_WAIT(bar_mma, mma_phase, kErrTimeoutMma);
        mma_phase ^= 1;
        tc_fence_after();
        const float GC = s_G[63];
        const float eGC = s_eG[63];

        // ---- A (rows of K K^T) and M (rows of Q K^T), masked before the exp
        {
            float v[32];
            tmem_ld32(tlane + T_KQ + 32 * hf, v);
            tmem_ld_wait();
            if (q4 < 2) {
                const int i = row;
                const float Gi = s_G[i], bi = s_beta[i];
                float a[32];
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const int j = 32 * hf + jj;
                    a[jj] = (j < i) ? bi * __expf(Gi - s_G[j]) * v[jj] : 0.f;
                }
                float4* dst = reinterpret_cast<float4*>(sA + i * LDA + 32 * hf);
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) dst[j4] = make_float4(a[4 * j4], a[4 * j4 + 1], a[4 * j4 + 2], a[4 * j4 + 3]);
            } else {
                const int i = row - 64;
                const float Gi = s_G[i];
                float m[32];
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const int j = 32 * hf + jj;
                    m[jj] = (j <= i) ? v[jj] * __expf(Gi - s_G[j]) : 0.f;
                }
                store_row_f16_sw128(smem + OFF_M, i, 4 * hf, m, 1.f);
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---- T = (I + A)^-1, then T diag(beta) and T diag(beta e^G) as f16 B operands
        chunk_tsolve(sA, sP, tid);
        {
            const int t = tid >> 2, part = tid & 3;
            const float* Tr = sA + t * LDA + 16 * part;
            float t1[16], t2[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int tp = 16 * part + e;
                const float tv = Tr[e];
                t1[e] = tv * s_beta[tp];
                t2[e] = t1[e] * s_eG[tp];
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                uint4 p1, p2;
                p1.x = pack_half2(t1[8 * j], t1[8 * j + 1]);
                p1.y = pack_half2(t1[8 * j + 2], t1[8 * j + 3]);
                p1.z = pack_half2(t1[8 * j + 4], t1[8 * j + 5]);
                p1.w = pack_half2(t1[8 * j + 6], t1[8 * j + 7]);
                p2.x = pack_half2(t2[8 * j], t2[8 * j + 1]);
                p2.y = pack_half2(t2[8 * j + 2], t2[8 * j + 3]);
                p2.z = pack_half2(t2[8 * j + 4], t2[8 * j + 5]);
                p2.w = pack_half2(t2[8 * j + 6], t2[8 * j + 7]);
                *reinterpret_cast<uint4*>(smem + OFF_T1 + sw128_chunk(t, 2 * part + j)) = p1;
                *reinterpret_cast<uint4*>(smem + OFF_T2 + sw128_chunk(t, 2 * part + j)) = p2;
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- MMA2: U~^T = V^T (T diag beta)^T ; MMA3: W^T = K^T (T diag(beta e^G))^T
        if (tid == 0) {
            // A / T are consumed: the residual tile of the next chunk can land.
            if (c + 1 < nchunks) {
                const int y = tok0 + C;
                mbar_arrive_expect_tx(bar_lo, LO_BYTES);
                tma_load_2d(smem + OFF_LO, &tmKl, kap * 128, y, bar_lo);
                tma_load_2d(smem + OFF_LO + 16384, &tmKl, kap * 128 + 64, y, bar_lo);
                tma_load_2d(smem + OFF_LO + 8192, &tmQl, kap * 128, y, bar_lo);
                tma_load_2d(smem + OFF_LO + 24576, &tmQl, kap * 128 + 64, y, bar_lo);
            }
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_f16(tbase + T_UT, sw128_desc(sbase + OFF_V + s * 2048, 8192, 1024),
                        sw128_desc(sbase + OFF_T1 + s * 32, 16, 1024), ID_AMN, s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_f16(tbase + T_WT, sw128_desc(aKQ + s * 2048, 16384, 1024),
                        sw128_desc(sbase + OFF_T2 + s * 32, 16, 1024), ID_AMN, s > 0);
            mma_commit(bar_mma);
        }
        CHUNK_WAIT(bar_mma, mma_phase, kErrTimeoutMma);
        mma_phase ^= 1;
        tc_fence_after();

        // V and the other K/Q buffer are free: fetch the next chunk's K, Q, V.
        if (tid == 0 && c + 1 < nchunks) {
            const uint32_t nxt = (c & 1) ? OFF_KQ0 : OFF_KQ1;
            const int y = tok0 + C;
            mbar_arrive_expect_tx(bar_kqv, KQV_BYTES);
            tma_load_2d(smem + nxt, &tmK, kap * 128, y, bar_kqv);
            tma_load_2d(smem + nxt + 16384, &tmK, kap * 128 + 64, y, bar_kqv);
            tma_load_2d(smem + nxt + 8192, &tmQ, kap * 128, y, bar_kqv);
            tma_load_2d(smem + nxt + 24576, &tmQ, kap * 128 + 64, y, bar_kqv);
            tma_load_2d(smem + OFF_V, &tmV, h * 128, y, bar_kqv);
            tma_load_2d(smem + OFF_V + 8192, &tmV, h * 128 + 64, y, bar_kqv);
        }

        // ---- W^T to shared memory (MN-major B operand: row k, 64 tokens)
        {
            float v[32];
            tmem_ld32(tlane + T_WT + 32 * hf, v);
            tmem_ld_wait();
            store_row_f16_sw128(smem + OFF_WT, row, 4 * hf, v, 1.f);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- MMA4: U^T = U~^T - S0 W^T ; MMA5: Oi^T = S0 Q^T
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint64_t a = sw128_desc(sbase + OFF_S + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
                mma_f16(tbase + T_UT, a, sw128_desc(sbase + OFF_WT + s * 2048, 8192, 1024), ID_NEG_BMN, 1);
            }
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                mma_f16(tbase + T_OI, sw128_desc(sbase + OFF_S + off, 16, 1024),
                        sw128_desc(aKQ + 8192 + off, 16, 1024), ID_KK, s > 0);
            }
            mma_commit(bar_mma);
        }
        CHUNK_WAIT(bar_mma, mma_phase, kErrTimeoutMma);
        mma_phase ^= 1;
        tc_fence_after();
        // W^T is consumed: the z tile of this chunk lands in its place.
        if (tid == 0) {
            mbar_arrive_expect_tx(bar_z, Z_BYTES);
            tma_load_2d(smem + OFF_Z, &tmZ, h * 128, tok0, bar_z);
        }

        // ---- U^T to shared memory, plain and scaled by e^{G_C - G_t}
        {
            float v[32];
            tmem_ld32(tlane + T_UT + 32 * hf, v);
            tmem_ld_wait();
            store_row_f16_sw128(smem + OFF_UT, row, 4 * hf, v, 1.f);
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) v[jj] *= __expf(GC - s_G[32 * hf + jj]);
            store_row_f16_sw128(smem + OFF_UTS, row, 4 * hf, v, 1.f);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- MMA6: dS = (U^T diag e^{G_C-G}) K ; MMA7: Oa^T = U^T M^T
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_f16(tbase + T_S, sw128_desc(sbase + OFF_UTS + s * 32, 16, 1024),
                        sw128_desc(aKQ + s * 2048, 16384, 1024), ID_DS, s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_f16(tbase + T_OA, sw128_desc(sbase + OFF_UT + s * 32, 16, 1024),
                        sw128_desc(sbase + OFF_M + s * 32, 16, 1024), ID_KK, s > 0);
            mma_commit(bar_mma);
        }
        CHUNK_WAIT(bar_mma, mma_phase, kErrTimeoutMma);
        mma_phase ^= 1;
        tc_fence_after();

        // ---- state update in registers, re-staged as f16 for the next chunk
        {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float d[32];
                tmem_ld32(tlane + T_S + 64 * hf + 32 * half, d);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) S[32 * half + j] = fmaf(eGC, S[32 * half + j], d[j]);
            }
            uint8_t* sS = smem + OFF_S + 16384 * hf;
            store_row_f16_sw128(sS, row, 0, S, 1.f);
            store_row_f16_sw128(sS, row, 4, S + 32, 1.f);
        }

        // ---- epilogue: o = e^G * Oi + Oa, gated RMSNorm over the 128 v channels
        CHUNK_WAIT(bar_z, c & 1, kErrTimeoutTma);
        {
            float o[32], oa[32];
            tmem_ld32(tlane + T_OI + 32 * hf, o);
            tmem_ld32(tlane + T_OA + 32 * hf, oa);
            tmem_ld_wait();
            float sq[32];
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
                o[jj] = fmaf(s_eG[32 * hf + jj], o[jj], oa[jj]);
                sq[jj] = o[jj] * o[jj];
            }
            const float part = warp_transpose_sum(sq, lane);
            s_red[q4 * 64 + 32 * hf + lane] = part;
            __syncthreads();
            if (tid < 64) {
                const float ms = (s_red[tid] + s_red[64 + tid] + s_red[128 + tid] + s_red[192 + tid]) * (1.0f / 128.0f);
                s_rstd[tid] = rsqrtf(ms + kEps);
            }
            __syncthreads();
            uint16_t* zt = reinterpret_cast<uint16_t*>(smem + OFF_Z);
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
                const int t = 32 * hf + jj;
                const float zv = bf16_bits_to_float(zt[t * 128 + row]);
                const float y = o[jj] * s_rstd[t] * wn * silu_f(zv);
                zt[t * 128 + row] = float_to_bf16_bits(y);
            }
        }
        __syncthreads();
        for (int idx = tid; idx < C * 16; idx += kThreads) {
            const int t = idx >> 4, cc = idx & 15;
            if (t < nv) {
                const uint4 v = *reinterpret_cast<const uint4*>(smem + OFF_Z + t * 256 + cc * 16);
                *reinterpret_cast<uint4*>(p.out + (size_t)(tok0 + t) * p.Vh * 128 + h * 128 + cc * 8) = v;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    if (!failed && p.final_state != nullptr) {
        float* dst = p.final_state + (((size_t)n * p.Vh + h) * 128 + row) * 128 + 64 * hf;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            reinterpret_cast<float4*>(dst)[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, TMEM_COLS);
}

#undef CHUNK_WAIT

}  // namespace gdn
