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
// One CTA owns one (row, value head) and walks its chunks in order, with two
// warp-specialised groups working on consecutive chunks at once:
//   * the prologue warpgroup (4 warps) does everything of chunk c+1 that does
//     not need the state: gates, MMA1 [K;Q]K^T (from f16 hi/lo parts:
//     hi.hi + hi.lo + lo.hi), the masked decay matrices A and M, the inverse
//     T = (I + A)^-1 (16 x 16 diagonal blocks on the CUDA cores, the merges on
//     the tensor cores in f32-accurate TF32), MMA2 U~^T = V^T (T diag beta)^T
//     and MMA3 W^T = K^T (T diag(beta e^G))^T, and issues the TMA loads;
//   * the state warpgroups (8 warps) run the chain of chunk c: MMA4
//     U^T = U~^T - S0 W^T and MMA5 Oi^T = S0 Q^T (S0 as f16 in shared memory),
//     U^T to f16 in TMEM (plain and scaled by e^{G_C - G}), the f32 state in
//     TMEM scaled by e^{G_C}, MMA6 S += (U^T diag e^{G_C-G}) K and MMA7
//     Oa^T = U^T (tril(QK^T)*E)^T with A read from TMEM, the f16 re-staging of
//     the state, and the gated-RMSNorm epilogue.
// Every contraction is a tcgen05.mma with M = 128 and an f32 accumulator in
// TMEM.  The groups hand buffers over with mbarriers; the buffers that both
// groups touch within one chunk are double-buffered.  Inputs come from the
// load-stage kernel as f16 tiles fetched with TMA.
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
    const uint16_t* z;        // bf16 [total][Vh*128]
    uint16_t* out;            // bf16 [total][Vh*128]
};

namespace chunk {
constexpr int C = 64;              // tokens per chunk
constexpr int kPThreads = 256;     // prologue warpgroups
constexpr int kSThreads = 256;     // state warpgroups
constexpr int kThreads = kPThreads + kSThreads;
constexpr int LDA = 68;            // f32 row stride of the A / T matrix (conflict-free float4 rows)
// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ0 = 0;        // [K rows 0-63 | Q rows 64-127] x k 0-63, then x k 64-127 (f16 hi parts)
constexpr uint32_t OFF_KQ1 = 32768;    // second buffer
constexpr uint32_t OFF_LO = 65536;     // same layout, f16 residuals; then A / T f32 and the T-solve scratch
constexpr uint32_t OFF_V = 98304;      // V [64 t][64 v] x 2 blocks
constexpr uint32_t OFF_WT = 114688;    // W^T f16 [128 k][64 t]
constexpr uint32_t OFF_Z = 131072;     // z bf16 [64 t][128], plain row-major
constexpr uint32_t OFF_S16 = 147456;   // S0 f16 [128 v][64 k] x 2 blocks
constexpr uint32_t OFF_T1 = 180224;    // T diag(beta) f16 [64][64]
constexpr uint32_t OFF_T2 = 188416;    // T diag(beta e^G) f16 [64][64]
constexpr uint32_t OFF_M0 = 196608;    // tril(Q K^T) * E f16 [64][64], two buffers
constexpr uint32_t OFF_M1 = 204800;
constexpr uint32_t OFF_MISC = 212992;
constexpr uint32_t MISC_BYTES = 4096;
constexpr uint32_t SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;  // + alignment slack
constexpr uint32_t OFF_A = OFF_LO;                       // f32 [64][LDA]
constexpr uint32_t OFF_TSCR = OFF_LO + 64 * LDA * 4;     // f32 scratch of the T-solve (32 x 36)
static_assert(64 * LDA * 4 + 32 * 36 * 4 <= 32768, "A/T and scratch must fit in the residual tile");
// misc: 0 barriers, 128 TMEM slot, 256 G[2][64], 768 e^G[2][64], 1280 e^{G_C-G}[2][64],
// 1792 beta[64], 2048 reductions [4][64], 3072 rstd[64], 3328 e^{G_C}[2]
// TMEM columns (f32, 128 lanes)
constexpr uint32_t T_KQ = 0, T_WT = 64, T_U0 = 128, T_U1 = 192, T_OI = 256, T_OA = 320, T_S = 384;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t KQV_BYTES = 6 * 8192;
constexpr uint32_t Z_BYTES = 64 * 128 * 2;
constexpr uint32_t LO_BYTES = 4 * 8192;
constexpr uint32_t ID_KK = idesc_f16_f32(128, 64, false, false, false);
constexpr uint32_t ID_AMN = idesc_f16_f32(128, 64, true, false, false);
constexpr uint32_t ID_NEG_BMN = idesc_f16_f32(128, 64, false, true, true);
constexpr uint32_t ID_DS = idesc_f16_f32(128, 128, false, true, false);
// mbarrier slots
constexpr int B_KQV = 0, B_LO = 1, B_P = 2, B_S = 3, B_PRO = 4, B_ST = 6, B_KQF = 8, B_Z = 10, B_WTF = 11;
constexpr int kBars = 12;
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
// stride LDA), by the threads of the prologue warpgroups (named barrier 1).
// The four 16 x 16 diagonal blocks are inverted by forward substitution on the
// CUDA cores; the off-diagonal blocks follow from the block inverse
// [[Ta, 0], [Y, Tb]] with Y = -Tb * L_ba * Ta, first for the 16-blocks (1,0)
// and (3,2), then for the 32-block (1,0), on the tensor cores (f32-accurate
// TF32 products).  sP: 32 x 36 f32 of scratch.
__device__ __forceinline__ void chunk_tsolve(float* sA, float* sP, int p) {
    using namespace chunk;
    const int warp = p >> 5, lane = p & 31;
    float x[16];
    const int b = p >> 4, c = p & 15;
    if (p < 64) {
        const float* Ab = sA + (16 * b) * LDA + 16 * b;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float s = 0.f;
#pragma unroll
            for (int m = 0; m < r; ++m) s = fmaf(Ab[r * LDA + m], x[m], s);
            x[r] = (r == c) ? 1.f : ((r < c) ? 0.f : -s);
        }
    }
    named_barrier_sync(1, kPThreads);
    if (p < 64) {
        float* Ab = sA + (16 * b) * LDA + 16 * b;
#pragma unroll
        for (int r = 0; r < 16; ++r) Ab[r * LDA + c] = x[r];
    }
    named_barrier_sync(1, kPThreads);
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
    named_barrier_sync(1, kPThreads);
    // 32-block merge: one 16 x 16 quadrant per warp (warps 0-3)
    const int mi = (warp >> 1) & 1, ni = warp & 1;
    float* X = sP;  // 32 x 32 scratch, stride 36
    if (warp < 4) {
        float acc[2][4] = {};
        warp_gemm_tf32x3<2, 4>(acc, sA + (32 + 16 * mi) * LDA, LDA, sA + 16 * ni, LDA, lane);
        warp_store_tile<2>(X + (16 * mi) * 36 + 16 * ni, 36, acc, 1.f, lane);
    }
    named_barrier_sync(1, kPThreads);  // X complete; every read of L_ba is done
    if (warp < 4) {
        float acc2[2][4] = {};
        warp_gemm_tf32x3<2, 4>(acc2, sA + (32 + 16 * mi) * LDA + 32, LDA, X + 16 * ni, 36, lane);
        warp_store_tile<2>(sA + (32 + 16 * mi) * LDA + 16 * ni, LDA, acc2, -1.f, lane);
    }
    named_barrier_sync(1, kPThreads);
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
    const int kap = h / (p.Vh / p.Kh);

    uint8_t* misc = smem + OFF_MISC;
    uint64_t* bars = reinterpret_cast<uint64_t*>(misc);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(misc + 128);
    float* s_G = reinterpret_cast<float*>(misc + 256);      // [2][64]
    float* s_eG = reinterpret_cast<float*>(misc + 768);     // [2][64]
    float* s_dec = reinterpret_cast<float*>(misc + 1280);   // [2][64]  e^{G_C - G_t}
    float* s_beta = reinterpret_cast<float*>(misc + 1792);  // [64]
    float* s_red = reinterpret_cast<float*>(misc + 2048);   // [4][64]
    float* s_rstd = reinterpret_cast<float*>(misc + 3072);  // [64]
    float* s_gC = reinterpret_cast<float*>(misc + 3328);    // [2]     e^{G_C}
    float* sA = reinterpret_cast<float*>(smem + OFF_A);
    float* sP = reinterpret_cast<float*>(smem + OFF_TSCR);

    int start, len;
    p.seq.bounds(n, start, len);
    const int nchunks = (len + C - 1) / C;

    if (tid == 0) {
        for (int i = 0; i < kBars; ++i) mbar_init(&bars[i], 1);
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

    auto load_kqv = [&](uint32_t kq_off, int y) {
        mbar_arrive_expect_tx(&bars[B_KQV], KQV_BYTES);
        tma_load_2d(smem + kq_off, &tmK, kap * 128, y, &bars[B_KQV]);
        tma_load_2d(smem + kq_off + 16384, &tmK, kap * 128 + 64, y, &bars[B_KQV]);
        tma_load_2d(smem + kq_off + 8192, &tmQ, kap * 128, y, &bars[B_KQV]);
        tma_load_2d(smem + kq_off + 24576, &tmQ, kap * 128 + 64, y, &bars[B_KQV]);
        tma_load_2d(smem + OFF_V, &tmV, h * 128, y, &bars[B_KQV]);
        tma_load_2d(smem + OFF_V + 8192, &tmV, h * 128 + 64, y, &bars[B_KQV]);
    };
    auto load_lo = [&](int y) {
        mbar_arrive_expect_tx(&bars[B_LO], LO_BYTES);
        tma_load_2d(smem + OFF_LO, &tmKl, kap * 128, y, &bars[B_LO]);
        tma_load_2d(smem + OFF_LO + 16384, &tmKl, kap * 128 + 64, y, &bars[B_LO]);
        tma_load_2d(smem + OFF_LO + 8192, &tmQl, kap * 128, y, &bars[B_LO]);
        tma_load_2d(smem + OFF_LO + 24576, &tmQl, kap * 128 + 64, y, &bars[B_LO]);
    };
    auto load_z = [&](int y) {
        mbar_arrive_expect_tx(&bars[B_Z], Z_BYTES);
        tma_load_2d(smem + OFF_Z, &tmZ, h * 128, y, &bars[B_Z]);
    };
    if (tid == 0 && nchunks > 0) {
        load_kqv(OFF_KQ0, start);
        load_lo(start);
        load_z(start);
    }
    bool broken = false;
    // every thread of the warp calls this; the warp is converged again on return
    auto wait = [&](int slot, uint32_t parity) {
        if (!broken && !mbar_wait(&bars[slot], parity)) {
            broken = true;
            record_error(kErrTimeoutTma);
        }
        __syncwarp();
    };

    if (warp < kPThreads / 32) {
        // =================================================================== prologue warpgroups
        const int pt = tid;
        const int pq = warp & 3;             // TMEM lane quarter
        const int phf = warp >> 2;           // column half
        const int prow = 32 * pq + lane;     // TMEM lane / matrix row of this thread
        const uint32_t tlane = tbase + (static_cast<uint32_t>(32 * pq) << 16);
        float g_next = 0.f, b_next = 0.f;
        if (pt < 64 && nchunks > 0 && pt < min(C, len)) {
            g_next = __ldg(p.Gs + (size_t)h * p.total + start + pt);
            b_next = __ldg(p.Bs + (size_t)h * p.total + start + pt);
        }
        uint32_t pphase = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            const int tok0 = start + c * C;
            const uint32_t kq_off = b ? OFF_KQ1 : OFF_KQ0;
            const uint32_t aKQ = sbase + kq_off;
            float* G = s_G + 64 * b;
            float* eG = s_eG + 64 * b;
            float* dec = s_dec + 64 * b;
            uint8_t* sM = smem + (b ? OFF_M1 : OFF_M0);
            uint8_t* sWt = smem + OFF_WT;
            const uint32_t T_U = b ? T_U1 : T_U0;
            // the state group must be done with chunk c-2's copies of these buffers
            if (c >= 2) wait(B_ST + b, ((c - 2) >> 1) & 1);

            // ---- gates: G = inclusive cumsum of g, e^G, beta, e^{G_C - G}
            if (pt < 64) {
                const float g = g_next, bt = b_next;
                const int nv1 = min(C, len - (c + 1) * C);  // tokens of the next chunk (<= 0: none)
                g_next = (pt < nv1) ? __ldg(p.Gs + (size_t)h * p.total + tok0 + C + pt) : 0.f;
                b_next = (pt < nv1) ? __ldg(p.Bs + (size_t)h * p.total + tok0 + C + pt) : 0.f;
                float x = g;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, o);
                    if (lane >= o) x += y;
                }
                G[pt] = x;
                s_beta[pt] = bt;
            }
            named_barrier_sync(1, kPThreads);
            float Gi = 0.f;
            if (pt < 64) Gi = G[pt] + ((pt >= 32) ? G[31] : 0.f);
            named_barrier_sync(1, kPThreads);
            if (pt < 64) {
                G[pt] = Gi;
                eG[pt] = expf(Gi);
            }
            named_barrier_sync(1, kPThreads);
            if (pt < 64) dec[pt] = expf(G[63] - G[pt]);
            if (pt == 0) s_gC[b] = expf(G[63]);
            __syncwarp();

            // ---- MMA1: [K;Q] K^T from hi/lo f16 parts
            wait(B_KQV, c & 1);
            wait(B_LO, c & 1);
            if (pt == 0) {
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
                    mma_f16(tbase + T_KQ, sw128_desc(aKQ + off, 16, 1024), sw128_desc(aLO + off, 16, 1024), ID_KK,
                            1);
                }
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                    mma_f16(tbase + T_KQ, sw128_desc(aLO + off, 16, 1024), sw128_desc(aKQ + off, 16, 1024), ID_KK,
                            1);
                }
                mma_commit(&bars[B_P]);
            }
            __syncwarp();
            wait(B_P, pphase);
            pphase ^= 1;
            tc_fence_after();

            // ---- A (rows of K K^T) and M (rows of Q K^T), masked before the exp
            {
                float v[32];
                tmem_ld32(tlane + T_KQ + 32 * phf, v);
                tmem_ld_wait();
                if (prow < 64) {
                    const int i = prow;
                    const float bi = s_beta[i], Gr = G[i];
                    float a[32];
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int j = 32 * phf + jj;
                        a[jj] = (j < i) ? bi * __expf(Gr - G[j]) * v[jj] : 0.f;
                    }
                    float4* dst = reinterpret_cast<float4*>(sA + i * LDA + 32 * phf);
#pragma unroll
                    for (int j4 = 0; j4 < 8; ++j4)
                        dst[j4] = make_float4(a[4 * j4], a[4 * j4 + 1], a[4 * j4 + 2], a[4 * j4 + 3]);
                } else {
                    const int i = prow - 64;
                    const float Gq = G[i];
                    float m[32];
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int j = 32 * phf + jj;
                        m[jj] = (j <= i) ? v[jj] * __expf(Gq - G[j]) : 0.f;
                    }
                    store_row_f16_sw128(sM, i, 4 * phf, m, 1.f);
                }
            }
            tc_fence_before();
            named_barrier_sync(1, kPThreads);

            // ---- T = (I + A)^-1, then T diag(beta) and T diag(beta e^G) as f16 B operands
            chunk_tsolve(sA, sP, pt);
            {
                const int t = pt >> 2, part = pt & 3;
                const float* Tr = sA + t * LDA + 16 * part;
                float t1[16], t2[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int tp = 16 * part + e;
                    t1[e] = Tr[e] * s_beta[tp];
                    t2[e] = t1[e] * eG[tp];
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
            named_barrier_sync(1, kPThreads);

            // ---- MMA2: U~^T = V^T (T diag beta)^T ; MMA3: W^T = K^T (T diag(beta e^G))^T
            if (pt == 0) {
                // A / T are consumed: the residual tile of the next chunk can land.
                if (c + 1 < nchunks) load_lo(tok0 + C);
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_f16(tbase + T_U, sw128_desc(sbase + OFF_V + s * 2048, 8192, 1024),
                            sw128_desc(sbase + OFF_T1 + s * 32, 16, 1024), ID_AMN, s > 0);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_f16(tbase + T_WT, sw128_desc(aKQ + s * 2048, 16384, 1024),
                            sw128_desc(sbase + OFF_T2 + s * 32, 16, 1024), ID_AMN, s > 0);
                mma_commit(&bars[B_P]);
            }
            __syncwarp();
            wait(B_P, pphase);
            pphase ^= 1;
            tc_fence_after();
            // V and the other K/Q buffer (once the state group has released it) take the next chunk.
            if (warp == 0 && c + 1 < nchunks) {
                if (c >= 1) wait(B_KQF + ((c - 1) & 1), ((c - 1) >> 1) & 1);
                if (pt == 0) load_kqv(b ? OFF_KQ0 : OFF_KQ1, tok0 + C);
                __syncwarp();
            }

            // ---- W^T to shared memory (MN-major B operand: row k, 64 tokens), once the
            //      state group's MMA4 of chunk c-1 has read the previous one
            if (c >= 1) wait(B_WTF, (c - 1) & 1);
            {
                float v[32];
                tmem_ld32(tlane + T_WT + 32 * phf, v);
                tmem_ld_wait();
                store_row_f16_sw128(sWt, prow, 4 * phf, v, 1.f);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_barrier_sync(1, kPThreads);
            if (pt == 0) mbar_arrive(&bars[B_PRO + b]);  // chunk c's prologue is ready
        }
    } else {
        // =================================================================== state warpgroups
        const int st = tid - kPThreads;         // 0..255
        const int sw = st >> 5;                 // 0..7
        const int q4 = sw & 3;                  // TMEM lane quarter (warp % 4)
        const int hf = sw >> 2;                 // column half
        const int row = 32 * q4 + lane;         // v row of the state / output channel
        const uint32_t tlane = tbase + (static_cast<uint32_t>(32 * q4) << 16);

        // initial state: f32 in TMEM (columns 64*hf .. +63 of this row), f16 copy in shared memory
        {
            const float* src =
                p.init_state ? p.init_state + (((size_t)n * p.Vh + h) * 128 + row) * 128 + 64 * hf : nullptr;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 f = src ? __ldg(reinterpret_cast<const float4*>(src + 32 * half) + j)
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
                    v[4 * j] = f.x;
                    v[4 * j + 1] = f.y;
                    v[4 * j + 2] = f.z;
                    v[4 * j + 3] = f.w;
                }
                uint32_t r[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(v[j]);
                tmem_st32(tlane + T_S + 64 * hf + 32 * half, r);
                store_row_f16_sw128(smem + OFF_S16 + 16384 * hf, row, 4 * half, v, 1.f);
            }
            tmem_st_wait();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        named_barrier_sync(2, kSThreads);

        const float wn = 1.0f + __ldg(p.norm_w + row);  // (1 + w) of this thread's v channel
        uint32_t sphase = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            const int tok0 = start + c * C;
            const int nv = min(C, len - c * C);
            const uint32_t aKQ = sbase + (b ? OFF_KQ1 : OFF_KQ0);
            const float* eG = s_eG + 64 * b;
            const float* dec = s_dec + 64 * b;
            const uint32_t aWt = sbase + OFF_WT;
            const uint32_t aM = sbase + (b ? OFF_M1 : OFF_M0);
            const uint32_t T_U = b ? T_U1 : T_U0;
            wait(B_PRO + b, (c >> 1) & 1);
            tc_fence_after();

            // ---- MMA4: U^T = U~^T - S0 W^T ; MMA5: Oi^T = S0 Q^T
            if (st == 0) {
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint64_t a = sw128_desc(sbase + OFF_S16 + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
                    mma_f16(tbase + T_U, a, sw128_desc(aWt + s * 2048, 8192, 1024), ID_NEG_BMN, 1);
                }
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                    mma_f16(tbase + T_OI, sw128_desc(sbase + OFF_S16 + off, 16, 1024),
                            sw128_desc(aKQ + 8192 + off, 16, 1024), ID_KK, s > 0);
                }
                mma_commit(&bars[B_S]);
            }
            __syncwarp();
            wait(B_S, sphase);
            sphase ^= 1;
            tc_fence_after();
            if (st == 0) mbar_arrive(&bars[B_WTF]);  // W^T of this chunk has been read
            __syncwarp();

            // ---- U^T to f16 in TMEM (plain, and scaled by e^{G_C - G_t}); state scaled by e^{G_C}
            {
                float u[32];
                tmem_ld32(tlane + T_U + 32 * hf, u);
                tmem_ld_wait();
                named_barrier_sync(2, kSThreads);  // every f32 U^T column is read before the f16 copies land
                uint32_t uh[16], us[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int t = 32 * hf + 2 * j;
                    uh[j] = pack_half2(u[2 * j], u[2 * j + 1]);
                    us[j] = pack_half2(u[2 * j] * dec[t], u[2 * j + 1] * dec[t + 1]);
                }
                tmem_st16(tlane + T_U + 16 * hf, uh);
                tmem_st16(tlane + T_U + 32 + 16 * hf, us);
                const float gC = s_gC[b];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float v[32];
                    tmem_ld32(tlane + T_S + 64 * hf + 32 * half, v);
                    tmem_ld_wait();
                    uint32_t r[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(gC * v[j]);
                    tmem_st32(tlane + T_S + 64 * hf + 32 * half, r);
                }
                tmem_st_wait();
            }
            tc_fence_before();
            named_barrier_sync(2, kSThreads);

            // ---- MMA6: S += (U^T diag e^{G_C-G}) K ; MMA7: Oa^T = U^T M^T  (A from TMEM)
            if (st == 0) {
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_f16_ta(tbase + T_S, tbase + T_U + 32 + 8 * s, sw128_desc(aKQ + s * 2048, 16384, 1024), ID_DS,
                               1);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_f16_ta(tbase + T_OA, tbase + T_U + 8 * s, sw128_desc(aM + s * 32, 16, 1024), ID_KK, s > 0);
                mma_commit(&bars[B_S]);
            }
            __syncwarp();
            wait(B_S, sphase);
            sphase ^= 1;
            tc_fence_after();
            if (st == 0) mbar_arrive(&bars[B_KQF + b]);  // K and Q of this chunk are no longer read
            __syncwarp();

            // ---- f16 copy of the new state for the next chunk's MMA4/5
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
                tmem_ld32(tlane + T_S + 64 * hf + 32 * half, v);
                tmem_ld_wait();
                store_row_f16_sw128(smem + OFF_S16 + 16384 * hf, row, 4 * half, v, 1.f);
            }

            // ---- epilogue: o = e^G * Oi + Oa, gated RMSNorm over the 128 v channels
            {
                float o[32], oa[32];
                tmem_ld32(tlane + T_OI + 32 * hf, o);
                tmem_ld32(tlane + T_OA + 32 * hf, oa);
                tmem_ld_wait();
                float sq[32];
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    o[jj] = fmaf(eG[32 * hf + jj], o[jj], oa[jj]);
                    sq[jj] = o[jj] * o[jj];
                }
                const float part = warp_transpose_sum(sq, lane);
                s_red[q4 * 64 + 32 * hf + lane] = part;
                named_barrier_sync(2, kSThreads);
                if (st < 64) {
                    const float ms =
                        (s_red[st] + s_red[64 + st] + s_red[128 + st] + s_red[192 + st]) * (1.0f / 128.0f);
                    s_rstd[st] = rsqrtf(ms + kEps);
                }
                named_barrier_sync(2, kSThreads);
                wait(B_Z, c & 1);
                const uint16_t* zt = reinterpret_cast<const uint16_t*>(smem + OFF_Z);
                uint16_t* op = p.out + (size_t)tok0 * p.Vh * 128 + h * 128 + row;
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const int t = 32 * hf + jj;
                    const float zv = bf16_bits_to_float(zt[t * 128 + row]);
                    const float y = o[jj] * s_rstd[t] * wn * silu_f(zv);
                    if (t < nv) op[(size_t)t * p.Vh * 128] = float_to_bf16_bits(y);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_barrier_sync(2, kSThreads);
            if (st == 0 && c + 1 < nchunks) load_z(tok0 + C);  // the z tile of the next chunk
            if (st == 0) mbar_arrive(&bars[B_ST + b]);  // chunk c's shared buffers are released
        }

        if (!broken && p.final_state != nullptr) {
            float* dst = p.final_state + (((size_t)n * p.Vh + h) * 128 + row) * 128 + 64 * hf;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
                tmem_ld32(tlane + T_S + 64 * hf + 32 * half, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    reinterpret_cast<float4*>(dst + 32 * half)[j] =
                        make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, TMEM_COLS);
}

}  // namespace gdn
