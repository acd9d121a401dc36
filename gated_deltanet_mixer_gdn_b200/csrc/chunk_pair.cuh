// Chunked prefill of the gated delta rule with the 128 value channels of a head
// split over a pair of CTAs (a thread-block cluster of two).
//
// The recurrence and the per-chunk record are those of chunk.cuh (Qwen3.8 27B
// model card, "Gated DeltaNet" bullet; chunk-64 WY form):
//     U   = T1 V - W S0^T,   O = Qs S0^T + M U,   S_C = e^{G_C} S0 + U^T K'.
// Row i of S (value channel i) evolves on its own: it uses v[i] and u[i] and the
// shared k, q and gates, nothing of the other rows.  So CTA r of the pair owns
// the channels [64 r, 64 r + 64) of the head, and each chunk's products and
// TMEM conversions are half those of the one-CTA form, which halves the
// sequential chain from one chunk to the next.  Only the gated RMSNorm, a mean
// over all 128 channels of a token, needs the partner: the two CTAs swap their
// 64 per-token sums of squares through distributed shared memory.
//
// The state is held transposed, S^T [128 k][64 v] f32 in TMEM (lane = k), so
// that every product keeps M = 128 with N = 64 value columns:
//     MMA-P  [U~ ; 0]  = [T1 ; 0] V          (zero rows: O starts cleared)
//     MMA-A  [U ; O]  += [-W ; Qs] S0^T      (S0^T f16 in shared memory)
//     MMA-S  S^T      += K'^T U              (U f16 in shared memory)
//     MMA7   [. ; O]  += [0 ; M] U
// with the tokens of a chunk in TMEM lanes 0-63 (U) and 64-127 (O).  Only
// MMA-A, the f16 copy of U, MMA-S and the f16 copy of the new state are on the
// chain; three accumulators let the epilogue trail the chain by up to two
// chunks.
#pragma once

#include "chunk.cuh"

namespace gdn {

namespace pair {
constexpr int C = 64;
constexpr int kConvWarps = 8;      // warps 0-7: TMEM -> f16 operands, state scaling
constexpr int kIssuerWarp = 24;    // tensor-core issue
constexpr int kLoaderWarp = 25;    // TMA and bulk loads of the chunk inputs
constexpr int kThreads = 26 * 32;
// warps 8-23: (warp & 3) >= 2 epilogue (TMEM lanes 64-127 hold O), else preparers
constexpr int kEThreads = 256;
// one input buffer; tiles f16 [64 rows][64] with 128-byte rows in the TMA 128B swizzle
constexpr uint32_t BUF_V = 0;         // V [t][64 v of this CTA] (TMA)
constexpr uint32_t BUF_T1 = 8192;     // T1 (record); with the zero tile after it, A = [T1 ; 0]
constexpr uint32_t BUF_ZERO = 16384;  // zeros (written once); with M after it, A = [0 ; M]
constexpr uint32_t BUF_M = 24576;     // M (record)
constexpr uint32_t BUF_WQ = 32768;    // per k block b at 16384 b: -W (record), then Q (TMA) scaled in place to Qs
constexpr uint32_t BUF_KP = 65536;    // K (TMA), 2 column blocks, scaled in place to K'
constexpr uint32_t BUF_DEC = 81920;   // f32 e^{G_C - G_t} [64], e^{G_t} [64], e^{G_C} (record)
constexpr uint32_t BUF_BYTES = 82944;
static_assert(BUF_DEC + wy::REC_DEC_BYTES <= BUF_BYTES, "input buffer");
constexpr uint32_t OFF_S16 = 2 * BUF_BYTES;     // S0^T f16 [128 k][64 v] (B of MMA-A)
constexpr uint32_t OFF_U16 = OFF_S16 + 16384;   // U f16 [64 t][64 v] (B of MMA-S and MMA7)
constexpr uint32_t OFF_ZT = OFF_U16 + 8192;     // 2 x z bf16 [64 t][64 v], swizzled; the output tiles
constexpr uint32_t OFF_MISC = OFF_ZT + 16384;
constexpr uint32_t MISC_BYTES = 3072;
constexpr uint32_t SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory");
// misc: 0 barriers, 256 TMEM slot, 512 sums of squares [4][64], 1536 rstd [64], 1792 the partner's sums [2][64]
constexpr uint32_t T_S = 0;    // S^T f32 [128 k][64 v]
constexpr uint32_t T_D = 64;   // + 64 * (c % 3): [U ; O] f32 of chunk c, 64 value columns
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t LD_BYTES = 9 * 8192 + wy::REC_DEC_BYTES;
constexpr uint32_t ZT_BYTES = 8192;
constexpr uint32_t ID_KM = idesc_f16_f32(128, 64, false, true, false);  // K-major A, MN-major B
constexpr uint32_t ID_S = idesc_f16_f32(128, 64, true, true, false);    // K'^T (MN-major) x U (MN-major)
// mbarrier slots
constexpr int B_LD = 0;     // + buffer: inputs landed
constexpr int B_A = 2;      // MMA-A complete
constexpr int B_UC = 3;     // U in f16 (one arrive per converter warp of lanes 0-63)
constexpr int B_SM = 4;     // MMA-S complete
constexpr int B_SC = 5;     // state in f16 (one arrive per converter warp)
constexpr int B_O = 6;      // + accumulator: MMA7 complete, O final
constexpr int B_E = 9;      // + accumulator: the epilogue has read O
constexpr int B_FREE = 12;  // + buffer: every MMA that reads the buffer is complete
constexpr int B_Z = 14;     // + z tile landed
constexpr int B_SS = 16;    // f32 state scaled by e^{G_C} (one arrive per converter warp)
constexpr int B_PREP = 17;  // + buffer: Qs and K' ready (one arrive per preparer warp)
constexpr int B_X = 19;     // + chunk parity: the partner's 64 per-token sums of squares landed (256 bytes)
constexpr int kBars = 21;
}  // namespace pair

__global__ void __launch_bounds__(pair::kThreads, 1)
    gdn_chunk_pair_kernel(const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmZ,
                          const __grid_constant__ CUtensorMap tmO, const ChunkParams p) {
    using namespace pair;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const uint32_t rank = cluster_ctarank();  // = blockIdx.x & 1 (clusters of two along x)
    const uint32_t peer = rank ^ 1u;
    const int h = blockIdx.x >> 1;
    const int v0 = 64 * (int)rank;  // first value channel of this CTA within the head
    const int n = p.order ? __ldg(p.order + blockIdx.y) : (int)blockIdx.y;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int kap = h / (p.Vh / p.Kh);
    const int q4 = warp & 3;  // TMEM lane quarter
    const uint32_t tlane = (static_cast<uint32_t>(32 * q4) << 16);

    uint8_t* misc = smem + OFF_MISC;
    uint64_t* bars = reinterpret_cast<uint64_t*>(misc);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(misc + 256);
    float* s_red = reinterpret_cast<float*>(misc + 512);    // [4][64]
    float* s_rstd = reinterpret_cast<float*>(misc + 1536);  // [64]
    float* s_x = reinterpret_cast<float*>(misc + 1792);     // [2][64], written by the partner
    uint8_t* sS16 = smem + OFF_S16;
    uint8_t* sU16 = smem + OFF_U16;

    int start, len;
    p.seq.bounds(n, start, len);
    const int srow = p.slots ? __ldg(p.slots + n) : n;  // state row
    // the chunks [cw, cw + nchunks) of the row; loop indices below count from cw
    const int cw = min(p.c0, (len + C - 1) / C);
    const int nchunks = max(0, (p.c1 < 0 ? (len + C - 1) / C : min(p.c1, (len + C - 1) / C)) - cw);
    const int cbase = (p.chunk_base ? __ldg(p.chunk_base + n) : n * ((p.seq.uniform_T + C - 1) / C)) + cw;
    start += cw * C;
    len -= cw * C;

    if (tid == 0) {
        for (int i = 0; i < kBars; ++i) {
            uint32_t cnt = 1;
            if (i == B_UC) cnt = 4;
            if (i == B_SC || i == B_SS || i == B_PREP || i == B_PREP + 1) cnt = 8;
            mbar_init(&bars[i], cnt);
        }
        fence_barrier_init();
        prefetch_tensormap(&tmV);
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmZ);
        prefetch_tensormap(&tmO);
    }
    // the zero tiles of both buffers
    for (int i = tid; i < 2 * 512; i += kThreads)
        *reinterpret_cast<uint4*>(smem + (i >> 9) * BUF_BYTES + BUF_ZERO + (i & 511) * 16) = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    if (warp == 0) {
        tmem_alloc(s_tmem, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync();  // the partner's barriers are initialised before any remote arrive
    const uint32_t tbase = *s_tmem;

    auto buf = [&](int c) { return smem + ((c & 1) ? BUF_BYTES : 0); };
    auto dacc = [&](int c) { return tbase + T_D + 64 * (uint32_t)(c % 3); };
    auto dec_of = [&](int c) { return reinterpret_cast<const float*>(buf(c) + BUF_DEC); };
    // (debug build: a record index out of range is recorded and record 0 is read instead)
    auto rec_of = [&](int c) {
        const bool ok = GDN_CHECK(cbase + c >= 0 && cbase + c < p.rec_chunks);
        return p.rec + (ok ? ((size_t)(cbase + c) * p.Vh + h) * wy::REC_BYTES : 0);
    };
    auto load_chunk = [&](int c) {
        uint8_t* B = buf(c);
        uint64_t* bar = &bars[B_LD + (c & 1)];
        const int y = start + c * C;
        (void)GDN_CHECK(y >= 0 && y < p.total);
        mbar_arrive_expect_tx(bar, LD_BYTES);
        tma_load_2d(B + BUF_V, &tmV, h * 128 + v0, y, bar);
        tma_load_2d(B + BUF_WQ + 8192, &tmQ, kap * 128, y, bar);
        tma_load_2d(B + BUF_WQ + 24576, &tmQ, kap * 128 + 64, y, bar);
        tma_load_2d(B + BUF_KP, &tmK, kap * 128, y, bar);
        tma_load_2d(B + BUF_KP + 8192, &tmK, kap * 128 + 64, y, bar);
        const uint8_t* r = rec_of(c);
        bulk_load(B + BUF_T1, r + wy::REC_T1, 8192, bar);
        bulk_load(B + BUF_WQ, r + wy::REC_MW, 8192, bar);
        bulk_load(B + BUF_WQ + 16384, r + wy::REC_MW + 8192, 8192, bar);
        bulk_load(B + BUF_M, r + wy::REC_M, 8192, bar);
        bulk_load(B + BUF_DEC, r + wy::REC_DEC, wy::REC_DEC_BYTES, bar);
    };
    auto prefetch_chunk = [&](int c) {
        const int y = start + c * C;
        prefetch_tma_2d(&tmV, h * 128 + v0, y);
        prefetch_tma_2d(&tmQ, kap * 128, y);
        prefetch_tma_2d(&tmQ, kap * 128 + 64, y);
        prefetch_tma_2d(&tmK, kap * 128, y);
        prefetch_tma_2d(&tmK, kap * 128 + 64, y);
        prefetch_l2(rec_of(c), wy::REC_BYTES);
    };
    auto load_z = [&](int c) {
        uint64_t* bar = &bars[B_Z + (c & 1)];
        mbar_arrive_expect_tx(bar, ZT_BYTES);
        tma_load_2d(smem + OFF_ZT + (c & 1) * ZT_BYTES, &tmZ, h * 128 + v0, start + c * C, bar);
    };
    bool broken = false;
    // every thread of the warp calls this; the warp is converged again on return
    auto wait = [&](int slot, uint32_t parity) {
        if (!broken && !mbar_wait(&bars[slot], parity)) {
            broken = true;
            record_error(kErrTimeoutTma);
        }
        __syncwarp();
    };
    // the same for a phase completed from the partner CTA (acquire at cluster scope)
    auto wait_cl = [&](int slot, uint32_t parity) {
        if (!broken && !mbar_wait_cluster(&bars[slot], parity)) {
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

    if (warp == kIssuerWarp) {
        // =================================================================== issue
        if (lane == 0 && nchunks > 0) {
            const uint32_t aS16 = smem_u32(sS16), aU16 = smem_u32(sU16);
            const uint64_t dK = sw128_desc(0, 16, 1024);    // K-major tiles
            const uint64_t dN = sw128_desc(0, 8192, 1024);  // MN-major tiles (two 64-wide blocks 8 KB apart)
            // MMA-P: [U~ ; 0] of chunk c into its accumulator (which also clears O)
            auto mma_P = [&](int c) {
                const uint32_t B = smem_u32(buf(c));
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_f16(dacc(c), desc_at(dK, B + BUF_T1 + s * 32), desc_at(dN, B + BUF_V + s * 2048), ID_KM, s > 0);
            };
            // the accumulator of chunk c is free once the epilogue has read O of chunk c - 3
            auto acc_ready = [&](int c) {
                return c < 3 || mbar_try_wait(smem_u32(&bars[B_E + c % 3]), (uint32_t)(c / 3 - 1) & 1u);
            };
            wait1(B_LD, 0);
            tc_fence_after();
            mma_P(0);
            for (int c = 0; c < nchunks; ++c) {
                const int b = c & 1;
                const uint32_t B = smem_u32(buf(c));
                const uint32_t d = dacc(c);
                wait1(B_SC, c & 1);               // S0^T of chunk c in f16
                wait1(B_PREP + b, (c >> 1) & 1);  // Qs and K' of chunk c
                tc_fence_after();
                // MMA-A: [U ; O] += [-W ; Qs] S0^T
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_f16(d, desc_at(dK, B + BUF_WQ + (s >> 2) * 16384 + (s & 3) * 32), desc_at(dN, aS16 + s * 2048),
                            ID_KM, 1);
                mma_commit(&bars[B_A]);
                // MMA-P of the next chunk now if its inputs are in and its accumulator is free,
                // else after MMA7
                bool p_next = c + 1 < nchunks;
                if (p_next && mbar_try_wait(smem_u32(&bars[B_LD + (b ^ 1)]), ((c + 1) >> 1) & 1) &&
                    acc_ready(c + 1)) {
                    tc_fence_after();
                    mma_P(c + 1);
                    p_next = false;
                }
                wait1(B_UC, c & 1);
                wait1(B_SS, c & 1);  // f32 state scaled by e^{G_C} of chunk c
                tc_fence_after();
                // MMA-S: S^T += K'^T U
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_f16(tbase + T_S, desc_at(dN, B + BUF_KP + s * 2048), desc_at(dN, aU16 + s * 2048), ID_S, 1);
                mma_commit(&bars[B_SM]);
                // MMA7: [. ; O] += [0 ; M] U
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_f16(d, desc_at(dK, B + BUF_ZERO + s * 32), desc_at(dN, aU16 + s * 2048), ID_KM, 1);
                mma_commit(&bars[B_O + c % 3]);
                mma_commit(&bars[B_FREE + b]);
                if (p_next) {
                    wait1(B_LD + (b ^ 1), ((c + 1) >> 1) & 1);
                    if (c + 1 >= 3) wait1(B_E + (c + 1) % 3, (uint32_t)((c + 1) / 3 - 1) & 1u);
                    tc_fence_after();
                    mma_P(c + 1);
                }
            }
        }
        __syncwarp();
    } else if (warp == kLoaderWarp) {
        // =================================================================== loads
        if (lane == 0 && nchunks > 0) {
            load_chunk(0);
            if (nchunks > 1) load_chunk(1);
            int issued = nchunks > 1 ? 2 : 1;  // chunks whose inputs were requested
            for (int c = 2; c < nchunks && c < 4; ++c) prefetch_chunk(c);
            // a buffer takes chunk c+2 once every MMA that reads chunk c is done
            for (int c = 0; c + 2 < nchunks; ++c) {
                wait1(B_FREE + (c & 1), (c >> 1) & 1);
                if (broken) break;  // no copy into a buffer that may still be read
                load_chunk(c + 2);
                issued = c + 3;
                if (c + 4 < nchunks) prefetch_chunk(c + 4);
            }
            // after a wait ran out, the CTA exits only once its copies in flight have landed
            // (the last request of each buffer; bounded)
            if (broken)
                for (int c = issued > 2 ? issued - 2 : 0; c < issued; ++c) mbar_wait(&bars[B_LD + (c & 1)], (c >> 1) & 1);
        }
        __syncwarp();
    } else if (warp < kConvWarps) {
        // =================================================================== converters
        const int ch = warp >> 2;         // value columns [32 ch, 32 ch + 32) of this CTA's 64
        const int k = 32 * q4 + lane;     // state column k (TMEM lane); a token of U for lanes 0-63
        const uint32_t tS = tbase + tlane + T_S + 32 * ch;
        // initial state: f16 copy for MMA-A, f32 scaled by the first chunk's e^{G_C}
        {
            float gC = 1.f;
            if (nchunks > 0) {
                wait(B_LD, 0);
                gC = dec_of(0)[128];
            }
            const float* src = p.init_state && GDN_CHECK(srow >= 0 && srow < p.state_rows)
                                   ? p.init_state + (((size_t)srow * p.Vh + h) * 128 + v0 + 32 * ch) * 128 + k
                                   : nullptr;
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = src ? __ldg(src + j * 128) : 0.f;
            store_row_f16_sw128(sS16, k, 4 * ch, v, 1.f);
            uint32_t r[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(gC * v[j]);
            tmem_st32(tS, r);
            tmem_st_wait();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&bars[B_SC]);
            mbar_arrive(&bars[B_SS]);
        }

        for (int c = 0; c < nchunks; ++c) {
            // ---- U to f16 (B of MMA-S and MMA7): lanes 0-63 of the accumulator
            if (q4 < 2) {
                wait(B_A, c & 1);
                tc_fence_after();
                float u[32];
                tmem_ld32(dacc(c) + tlane + 32 * ch, u);
                tmem_ld_wait();
                store_row_f16_sw128(sU16, k, 4 * ch, u, 1.f);
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_UC]);
            }
            // ---- the new state: f16 copy for the next MMA-A first, then the f32 state
            // scaled by the next e^{G_C} (needed only by the next MMA-S)
            wait(B_SM, c & 1);
            tc_fence_after();
            if (c + 1 < nchunks) {
                float v[32];
                tmem_ld32(tS, v);
                tmem_ld_wait();
                store_row_f16_sw128(sS16, k, 4 * ch, v, 1.f);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_SC]);
                wait(B_LD + ((c + 1) & 1), ((c + 1) >> 1) & 1);
                const float gC = dec_of(c + 1)[128];
                uint32_t r[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(gC * v[j]);
                tmem_st32(tS, r);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_SS]);
            }
        }

        if (!broken && p.final_state != nullptr && GDN_CHECK(srow >= 0 && srow < p.state_rows)) {
            float v[32];
            tmem_ld32(tS, v);
            tmem_ld_wait();
            float* dst = p.final_state + (((size_t)srow * p.Vh + h) * 128 + v0 + 32 * ch) * 128 + k;
#pragma unroll
            for (int j = 0; j < 32; ++j) dst[j * 128] = v[j];
        }
    } else if ((warp & 3) >= 2) {
        // =================================================================== epilogue
        const int e = (warp - 8) >> 2;       // value columns [16 e, 16 e + 16) of this CTA's 64
        const int t = 32 * (q4 - 2) + lane;  // token of the chunk (O row 64 + t)
        const bool lead = e == 0;            // warps of the per-token sums and the exchange
        const bool io = lead && t == 0;      // owner of the z loads and the output stores
        float wn[16];                        // (1 + w) of this thread's value channels
#pragma unroll
        for (int j = 0; j < 16; ++j) wn[j] = 1.0f + __ldg(p.norm_w + v0 + 16 * e + j);
        if (io && nchunks > 0) load_z(0);
        __syncwarp();
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            const int tok0 = start + c * C;
            const int nv = min(C, len - c * C);
            // z of chunk c+1 into the other tile, once the output of chunk c-1 has left it
            if (io && c + 1 < nchunks) {
                bulk_wait_read_all();
                load_z(c + 1);
            }
            __syncwarp();
            wait(B_O + c % 3, (uint32_t)(c / 3) & 1u);
            tc_fence_after();
            float o[16];
            tmem_ld16(dacc(c) + tlane + 16 * e, o);
            tmem_ld_wait();
            tc_fence_before();
            {
                float sq = 0.f;
#pragma unroll
                for (int j = 0; j < 16; ++j) sq = fmaf(o[j], o[j], sq);
                s_red[64 * e + t] = sq;
            }
            named_barrier_sync(3, kEThreads);
            if (io) mbar_arrive(&bars[B_E + c % 3]);  // the accumulator may take chunk c+3
            if (lead) {
                // this CTA's sum over its 64 channels to the partner (an asynchronous store that
                // completes bytes of the partner's barrier for chunk c); the partner's back.  A
                // barrier's next phase is armed here only after this thread saw its last one complete.
                const float loc = (s_red[t] + s_red[64 + t]) + (s_red[128 + t] + s_red[192 + t]);
                if (t == 0) mbar_arrive_expect_tx(&bars[B_X + b], 64 * 4);
                st_async_remote_f32(s_x + 64 * b + t, &bars[B_X + b], peer, loc);
                wait_cl(B_X + b, (c >> 1) & 1);
                // (a + b is exact-commutative, so both CTAs get the same rstd bits)
                s_rstd[t] = rsqrtf((loc + s_x[64 * b + t]) * (1.0f / 128.0f) + kEps);
            }
            named_barrier_sync(3, kEThreads);
            wait(B_Z + b, (c >> 1) & 1);
            uint8_t* zt = smem + OFF_ZT + b * ZT_BYTES;
            const float rs = s_rstd[t];
            {
                const uint4 z0 = *reinterpret_cast<const uint4*>(zt + sw128_chunk(t, 2 * e));
                const uint4 z1 = *reinterpret_cast<const uint4*>(zt + sw128_chunk(t, 2 * e + 1));
                const uint32_t zw[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float za = bf16_bits_to_float(static_cast<uint16_t>(zw[j] & 0xffffu));
                    const float zb = bf16_bits_to_float(static_cast<uint16_t>(zw[j] >> 16));
                    o[2 * j] = o[2 * j] * rs * wn[2 * j] * silu_tanh(za);
                    o[2 * j + 1] = o[2 * j + 1] * rs * wn[2 * j + 1] * silu_tanh(zb);
                }
            }
            uint32_t yb[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) yb[j] = pack_bf16x2(o[2 * j], o[2 * j + 1]);
            const uint4 y0 = make_uint4(yb[0], yb[1], yb[2], yb[3]), y1 = make_uint4(yb[4], yb[5], yb[6], yb[7]);
            // a full chunk is written over its z tile and leaves by one TMA store; a ragged
            // last chunk is stored directly (the rows past it belong to the next sequence)
            const bool full = (nv == C);
            if (full) {
                *reinterpret_cast<uint4*>(zt + sw128_chunk(t, 2 * e)) = y0;
                *reinterpret_cast<uint4*>(zt + sw128_chunk(t, 2 * e + 1)) = y1;
                fence_proxy_async_smem();
            } else if (t < nv && GDN_CHECK(tok0 + t < p.total)) {
                uint4* op = reinterpret_cast<uint4*>(p.out + (size_t)(tok0 + t) * p.Vh * 128 + h * 128 + v0 + 16 * e);
                op[0] = y0;
                op[1] = y1;
            }
            named_barrier_sync(3, kEThreads);
            if (io && full) {
                tma_store_2d(&tmO, zt, h * 128 + v0, tok0);
                bulk_commit();
            }
            __syncwarp();
        }
        if (io) {
            bulk_wait_all();
            // after a wait ran out, the z tiles in flight land before the CTA exits (bounded)
            if (broken)
                for (int k = nchunks > 2 ? nchunks - 2 : 0; k < nchunks; ++k) mbar_wait(&bars[B_Z + (k & 1)], (k >> 1) & 1);
        }
    } else {
        // =================================================================== preparers
        // Qs = diag(e^G) Q and K' = diag(e^{G_C - G}) K, in place; one row of 64 k per thread
        const int pt = (((warp - 8) >> 2) * 2 + (warp & 1)) * 32 + lane;  // 0..255
        const int which = pt >> 7;  // 0: Q rows, 1: K rows
        const int blk = (pt >> 6) & 1;
        const int t = pt & 63;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            wait(B_LD + b, (c >> 1) & 1);
            uint8_t* B = buf(c);
            const float sc = dec_of(c)[which ? t : 64 + t];
            uint8_t* tile = which ? B + BUF_KP + blk * 8192 : B + BUF_WQ + 8192 + blk * 16384;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                uint4* q = reinterpret_cast<uint4*>(tile + sw128_chunk(t, cc));
                uint4 v = *q;
                uint32_t* u = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[x]));
                    u[x] = pack_half2(f.x * sc, f.y * sc);
                }
                *q = v;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_PREP + b]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, TMEM_COLS);
    // no CTA of the pair exits while its partner may still write to its shared memory
    cluster_sync();
}

}  // namespace gdn
