// C ABI of the Gated DeltaNet mixer (declared in include/gdn.h): argument
// checks, workspace carving, TMA descriptor set-up and kernel launches.
// This is the library's only translation unit; the kernels are included.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/gdn.h"
#include "chunk.cuh"
#include "chunk_pair.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "gemm.cuh"
#include "inproj.cuh"
#include "prep.cuh"

namespace {

using namespace gdn;

// An NVTX range over one ABI call (named after the entry point), so host timelines of a
// profiler show each call and the launches it enqueued; free when no tool is attached.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(const gdn_dims* d) {
    if (d == nullptr) return GDN_ERR_INVALID_ARG;
    if (d->num_k_heads <= 0 || d->num_v_heads <= 0) return GDN_ERR_INVALID_ARG;
    if (d->head_dim != 128 || d->conv_width != 4) return GDN_ERR_UNSUPPORTED;
    if (d->num_v_heads % d->num_k_heads != 0) return GDN_ERR_UNSUPPORTED;
    if (d->num_v_heads / d->num_k_heads > 8) return GDN_ERR_UNSUPPORTED;
    if (d->num_v_heads > 1024 || d->num_k_heads > 1024) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

int check_weights(const gdn_weights* w) {
    if (w == nullptr || w->conv_w == nullptr || w->A_log == nullptr || w->dt_bias == nullptr || w->norm_w == nullptr)
        return GDN_ERR_INVALID_ARG;
    if (!aligned16(w->conv_w) || !aligned16(w->norm_w)) return GDN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(w->A_log) & 3u) || (reinterpret_cast<uintptr_t>(w->dt_bias) & 3u))
        return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

int check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return GDN_ERR_CUDA;
    return major == 10 ? GDN_OK : GDN_ERR_UNSUPPORTED;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D row-major map over [rows][cols] 16-bit elements, box {box_cols, box_rows}.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t cols, uint64_t rows, uint32_t box_cols,
              uint32_t box_rows, CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

struct Workspace {
    size_t off_q, off_k, off_ql, off_kl, off_v, off_g, off_b, off_cb, off_rec, bytes;
};

// Chunks over all rows: exact for uniform rows, and an upper bound for N rows
// of `total` tokens in all (each row adds at most one partial chunk).
int64_t chunk_bound(int64_t N, int64_t total) { return (total + 63 * N) / 64; }

Workspace plan_workspace(const gdn_dims* d, int64_t total, int64_t N, int64_t nchunks) {
    Workspace w{};
    const size_t qk = (size_t)total * d->num_k_heads * 128 * 2;
    const size_t vv = (size_t)total * d->num_v_heads * 128 * 2;
    const size_t gb = (size_t)total * d->num_v_heads * 4;
    w.off_q = 0;
    w.off_k = align_up(qk);
    w.off_ql = w.off_k + align_up(qk);
    w.off_kl = w.off_ql + align_up(qk);
    w.off_v = w.off_kl + align_up(qk);
    w.off_g = w.off_v + align_up(vv);
    w.off_b = w.off_g + align_up(gb);
    w.off_cb = w.off_b + align_up(gb);
    w.off_rec = w.off_cb + align_up((size_t)(2 * N + 1) * 4);  // chunk bases [N+1], then the row order [N]
    w.bytes = w.off_rec + align_up((size_t)nchunks * d->num_v_heads * wy::REC_BYTES);
    return w;
}

// Internal streams of the overlapped dense prefill, one set per device: the
// recurrence runs on a high-priority stream while the load stage and the WY
// records of the next segment run on a low-priority one.  Created on the
// first overlapped call on the device.
constexpr int kMaxSegments = 8;
struct SideStreams {
    bool ready = false;
    cudaStream_t prod = nullptr, chain = nullptr, tail = nullptr;  // priorities: chain > prod > tail
    cudaEvent_t fork = nullptr, prod_done = nullptr, chain_done = nullptr, tail_done = nullptr;
    cudaEvent_t seg[kMaxSegments] = {};   // WY records of a segment written (prod -> chain)
    cudaEvent_t rec[kMaxSegments] = {};   // recurrence of a segment done (chain -> prod)
};
std::mutex g_side_mu;
SideStreams g_side[kMaxDevices];

int side_streams(int dev, SideStreams** out) {
    if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_UNSUPPORTED;
    SideStreams& st = g_side[dev];
    if (!st.ready) {
        int least = 0, greatest = 0;
        if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) return GDN_ERR_CUDA;
        // (numerically lower is higher priority; with a single level all three are equal)
        const int middle = greatest < least ? greatest + 1 : greatest;
        if (cudaStreamCreateWithPriority(&st.prod, cudaStreamNonBlocking, middle) != cudaSuccess ||
            cudaStreamCreateWithPriority(&st.chain, cudaStreamNonBlocking, greatest) != cudaSuccess ||
            cudaStreamCreateWithPriority(&st.tail, cudaStreamNonBlocking, least) != cudaSuccess)
            return GDN_ERR_CUDA;
        cudaEvent_t* evs[4] = {&st.fork, &st.prod_done, &st.chain_done, &st.tail_done};
        for (cudaEvent_t* e : evs)
            if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return GDN_ERR_CUDA;
        for (auto& e : st.seg)
            if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return GDN_ERR_CUDA;
        for (auto& e : st.rec)
            if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return GDN_ERR_CUDA;
        st.ready = true;
    }
    *out = &st;
    return GDN_OK;
}

// Dynamic shared memory opt-in of a kernel (the attribute belongs to the device's context):
// once per kernel and device, under a lock.
int smem_optin(const void* kernel_fn, uint32_t bytes) {
    static std::mutex mu;
    static std::vector<std::pair<const void*, int>> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    for (auto& d : done)
        if (d.first == kernel_fn && d.second == dev) return GDN_OK;
    if (cudaFuncSetAttribute(kernel_fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return GDN_ERR_CUDA;
    done.emplace_back(kernel_fn, dev);
    return GDN_OK;
}

// The load stage fused into the in_proj GEMM: the hidden states and the
// stacked in_proj weights go in; the staged operands, z and the rows' last
// pre-conv tokens come out (z and the latter into workspace buffers).
struct FusedLoad {
    const uint16_t* x;     // bf16 [total][hidden]
    const uint16_t* w_in;  // bf16 [C + Vh*128 + 2*Vh][hidden]
    int hidden;
    uint16_t* z;           // bf16 [total][Vh*128]
    float* conv_last;      // f32 [N][3][C]
};

// out_proj after the mixer (gdn_prefill_out): out[t] = y[t] w_out^T for every token t,
// y being the mixer's gated-norm output.
struct OutProjTail {
    const uint16_t* w_out;  // bf16 [hidden][Vh*128]
    int hidden;
    uint16_t* out;          // bf16 [tokens][hidden]
};

int gemm_launch(const uint16_t* A, const uint16_t* W, struct GemmParams gp, cudaStream_t stream);

// out_proj of tokens [t0, t1) of the call (rows of y and of out).
int out_proj_range(const OutProjTail& op, const uint16_t* y, int VD, int64_t t0, int64_t t1, cudaStream_t st) {
    if (t1 <= t0) return GDN_OK;
    GemmParams gp{};
    gp.M = (int)(t1 - t0);
    gp.N = op.hidden;
    gp.K = VD;
    gp.nseg = 1;
    gp.seg[0] = GemmSegment{0, op.hidden, op.out + t0 * op.hidden};
    return gemm_launch(y + t0 * VD, op.w_out, gp, st);
}

// Segment plan of the overlapped dense prefill.  The load stage runs over all
// tokens first; segment 0's WY records run on every SM; after that, the recurrence
// of segment k (one CTA per row and value head) runs beside the WY records of
// segment k+1 on the remaining SMs.  The plan is picked on the host by simulating
// candidate plans with a cost model of this library's kernels measured on B200: a
// WY launch takes about 11.2 us per wave of tasks (a task: one chunk, one q/k head,
// up to 3 of its value heads) plus 4 us; a recurrence launch about 9.5 us plus 2.3 us
// per chunk (the WY figure as measured beside a running recurrence; erring slow keeps
// the recurrence from waiting).  Candidates: segment sizes growing or shrinking
// geometrically (s_k = s_0 rho^k: rho > 1 lets the recurrence start early when it
// bounds the call, rho < 1 runs most WY records on every SM first when they bound
// it), 2..kMaxSegments segments of at least one chunk, and the plain schedule.
// (Running the load stage per segment on the WY stream as well was measured no
// faster at one row and slower at two.)
namespace seg_model {
constexpr double kWaveUs = 11.2, kWyFixedUs = 4.0, kChainFixedUs = 9.5;
constexpr double kChainChunkUs = 2.3, kPairChainChunkUs = 1.9;  // one CTA per head; CTA pairs
}

// The recurrence runs on CTA pairs (each 64 of a head's value channels, a shorter per-chunk
// chain) when the pairs fit in one wave of SMs; with more rows one CTA per head does more work
// per SM (measured: 8 packed rows 0.60 ms against 0.87 ms on pairs, 2 x 65,536 tokens 2.28
// against 3.62 ms; one row of 8192 tokens 0.297 ms against 0.242 ms).
bool use_pair(int N, int Vh, int nsm) { return 2 * (int64_t)N * Vh <= nsm; }

struct SegPlan {
    int S = 1;  // segments (1: the plain schedule on the caller's stream)
    int cs[kMaxSegments + 1] = {};
};

// Time from the end of the load stage to the end of the last recurrence launch.
double simulate_plan(const SegPlan& pl, int tasks_per_chunk, int nsm, int chain_ctas, double chunk_us) {
    using namespace seg_model;
    const int P = pl.S > 1 ? nsm - chain_ctas : nsm;  // SMs of the WY stream beside a running recurrence
    auto wy_us = [&](int chunks, int sms) {
        const int64_t tasks = (int64_t)chunks * tasks_per_chunk;
        return kWaveUs * (double)((tasks + sms - 1) / sms) + kWyFixedUs;
    };
    double wy_end = wy_us(pl.cs[1], nsm), chain_end = 0.0;
    for (int k = 0; k < pl.S; ++k) {
        const double start = chain_end > wy_end ? chain_end : wy_end;
        chain_end = start + kChainFixedUs + chunk_us * (pl.cs[k + 1] - pl.cs[k]);
        if (k + 1 < pl.S) wy_end += wy_us(pl.cs[k + 2] - pl.cs[k + 1], P);
    }
    return chain_end;
}

// The plan for N dense rows of T tokens: overlap needs a recurrence that leaves at least
// 32 SMs to the WY records and rows of at least 16 chunks.
SegPlan dense_plan(int Kh, int Vh, int N, int T, int nsm, bool pair) {
    const int per = (T + 63) / 64;
    SegPlan best;
    best.cs[1] = per;
    const int chain_ctas = (pair ? 2 : 1) * N * Vh;
    const double chunk_us = pair ? seg_model::kPairChainChunkUs : seg_model::kChainChunkUs;
    if (chain_ctas + 32 > nsm || per < 16) return best;
    const int tasks_per_chunk = N * Kh * ((Vh / Kh + wy::kHeads - 1) / wy::kHeads);
    double best_t = simulate_plan(best, tasks_per_chunk, nsm, chain_ctas, chunk_us);
    static const double kRho[] = {0.2, 0.3, 0.4, 0.5, 0.6, 0.7, 0.8, 0.9, 1.0, 1.1, 1.2, 1.35, 1.5, 1.75, 2.0};
    const int max_S = per < kMaxSegments ? per : kMaxSegments;
    for (int S = 2; S <= max_S; ++S) {
        for (double rho : kRho) {
            SegPlan c;
            c.S = S;
            double total = 0.0, f = 1.0;
            for (int k = 0; k < S; ++k, f *= rho) total += f;
            double acc = 0.0;
            f = 1.0;
            for (int k = 1; k <= S; ++k, f *= rho) {
                acc += f / total * per;
                const int v = (int)(acc + 0.5);
                const int lo = c.cs[k - 1] + 1, hi = per - (S - k);  // every segment keeps at least one chunk
                c.cs[k] = v < lo ? lo : (v > hi ? hi : v);
            }
            c.cs[S] = per;
            const double t = simulate_plan(c, tasks_per_chunk, nsm, chain_ctas, chunk_us);
            if (t < best_t) {
                best_t = t;
                best = c;
            }
        }
    }
    return best;
}

// Kernels one dense call launches under a plan: the load stage (or the fused in_proj GEMM),
// the history writer, then WY records and recurrence per segment.
int plan_launches(const SegPlan& pl) { return 2 + 2 * pl.S; }

// Everything one prefill call launches, with the workspace carved and the
// tensor maps built once.
struct PrefillPlan {
    int Kh, Vh, C, N, uniform_T, total, nsm;
    SeqIndex seq;
    const gdn_weights* w;
    const uint16_t *qkv, *a, *b;
    const float* init_conv;
    float* final_conv;
    uint16_t* out;
    const float* norm_w;
    const int* slots;  // state / history row of each packed row, or nullptr
    const FusedLoad* fused;  // load stage inside the in_proj GEMM (dense rows), or nullptr
    __half *Qs, *Ks, *Ql, *Kl, *Vs;
    float *Gs, *Bs;
    int* chunk_base;
    int* order;  // recurrence row order (packed rows), or nullptr
    uint8_t* rec;
    int rec_chunks;  // chunks the record array holds
    int state_rows;  // rows of the state / history arrays (the pool's, with slots)
    bool pair;       // recurrence on CTA pairs (64 value channels each), else one CTA per head
    CUtensorMap mK, mQ, mKl, mQl, mV, mZ, mO;

    int prep(int tok_begin, int tok_end, cudaStream_t st) const {
        if (tok_end <= tok_begin) return GDN_OK;
        if (fused != nullptr) return fused_prep(st);  // always the whole range
        PrepParams pp{};
        pp.Kh = Kh;
        pp.Vh = Vh;
        pp.C = C;
        pp.total = total;
        pp.tok_begin = tok_begin;
        pp.tok_end = tok_end;
        pp.seq = seq;
        pp.qkv = qkv;
        pp.a = a;
        pp.b = b;
        pp.conv_w = w->conv_w;
        pp.A_log = w->A_log;
        pp.dt_bias = w->dt_bias;
        pp.init_conv = init_conv;
        pp.slots = slots;
        pp.Qs = Qs;
        pp.Ks = Ks;
        pp.Ql = Ql;
        pp.Kl = Kl;
        pp.Vs = Vs;
        pp.Gs = Gs;
        pp.Bs = Bs;
        CUtensorMap mX;  // the CTAs' input rows x 256-channel boxes (rows outside the tensor read as zero)
        if (!make_map(&mX, qkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)C, (uint64_t)total, kPrepBox, kPrepRows,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
            return GDN_ERR_CUDA;
        int rc = smem_optin(reinterpret_cast<const void*>(gdn_prep_kernel), kPrepSmem);
        if (rc != GDN_OK) return rc;
        dim3 grid((tok_end - tok_begin + kPrepTokens - 1) / kPrepTokens, (2 * Kh + Vh + kPrepSlots - 1) / kPrepSlots);
        gdn_prep_kernel<<<grid, 256, kPrepSmem, st>>>(mX, pp);
        return cuda_status(cudaGetLastError());
    }
    // in_proj + load stage over all tokens: 128-row tiles advancing by 125 tokens
    int fused_prep(cudaStream_t st) const {
        GemmParams gp{};
        gp.M = total;
        gp.N = C + Vh * 128 + 2 * Vh;
        gp.K = fused->hidden;
        FusedPrep f{};
        f.Kh = Kh;
        f.Vh = Vh;
        f.T = uniform_T;
        f.cu = seq.cu;
        f.N = N;
        f.conv_w = w->conv_w;
        f.A_log = w->A_log;
        f.dt_bias = w->dt_bias;
        f.init_conv = init_conv;
        f.Qs = Qs;
        f.Ks = Ks;
        f.Ql = Ql;
        f.Kl = Kl;
        f.Vs = Vs;
        f.Gs = Gs;
        f.Bs = Bs;
        f.z = fused->z;
        f.conv_last = fused->conv_last;
        CUtensorMap mA, mW;
        if (!make_map(&mA, fused->x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)gp.K, (uint64_t)gp.M, gemm::BK,
                      gemm::BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&mW, fused->w_in, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)gp.K, (uint64_t)gp.N, gemm::BK,
                      gemm::BN, CU_TENSOR_MAP_SWIZZLE_128B))
            return GDN_ERR_CUDA;
        int rc = smem_optin(reinterpret_cast<const void*>(gdn_gemm_kernel<1>), gemm::SMEM_BYTES);
        if (rc != GDN_OK) return rc;
        const int64_t ntiles = (int64_t)((gp.M + gemm::BM - 4) / (gemm::BM - 3)) * ((gp.N + gemm::BN - 1) / gemm::BN);
        const int grid = (int)(ntiles < nsm ? ntiles : nsm);
        gdn_gemm_kernel<1><<<grid, gemm::kThreads, gemm::SMEM_BYTES, st>>>(mA, mW, gp, f);
        return cuda_status(cudaGetLastError());
    }
    int conv_out(cudaStream_t st) const {
        if (final_conv == nullptr) return GDN_OK;
        if (fused != nullptr) {  // the rows' last tokens, staged by the fused load stage, and the history
            dim3 grid((C + 255) / 256, N);
            gdn_conv_merge_kernel<<<grid, 256, 0, st>>>(seq, C, fused->conv_last, init_conv, final_conv);
            return cuda_status(cudaGetLastError());
        }
        ConvOutParams cp{};
        cp.C = C;
        cp.N = N;
        cp.total = total;
        cp.seq = seq;
        cp.qkv = qkv;
        cp.init_conv = init_conv;
        cp.final_conv = final_conv;
        cp.slots = slots;
        dim3 grid((C + 255) / 256, N);
        gdn_conv_out_kernel<<<grid, 256, 0, st>>>(cp);
        return cuda_status(cudaGetLastError());
    }
    // WY records of nch chunks: all of them (win 0), or the window [c0, c0 + win) of every uniform row
    int wy_records(int64_t nch, int c0, int win, int grid_cap, cudaStream_t st) const {
        if (nch <= 0) return GDN_OK;
        WyParams wp{};
        wp.Kh = Kh;
        wp.Vh = Vh;
        wp.total = total;
        wp.seq = seq;
        wp.chunk_base = chunk_base;
        wp.nchunks = (int)nch;
        wp.c0 = c0;
        wp.win = win;
        wp.Gs = Gs;
        wp.Bs = Bs;
        wp.rec = rec;
        wp.rec_chunks = rec_chunks;
        int rc = smem_optin(reinterpret_cast<const void*>(gdn_wy_kernel), wy::SMEM_BYTES);
        if (rc != GDN_OK) return rc;
        const int ratio = Vh / Kh;
        const int64_t ntasks = nch * Kh * ((ratio + wy::kHeads - 1) / wy::kHeads);
        const int grid = (int)(ntasks < grid_cap ? ntasks : grid_cap);
        gdn_wy_kernel<<<grid, wy::kThreads, wy::SMEM_BYTES, st>>>(mK, mQ, mKl, mQl, wp);
        return cuda_status(cudaGetLastError());
    }
    // the recurrence over the chunk window [c0, c1) of every row (c1 < 0: to the end)
    int recurrence(int c0, int c1, const float* init_state, float* final_state, cudaStream_t st) const {
        ChunkParams cp{};
        cp.Kh = Kh;
        cp.Vh = Vh;
        cp.total = total;
        cp.seq = seq;
        cp.chunk_base = chunk_base;
        cp.order = order;
        cp.rec = rec;
        cp.init_state = init_state;
        cp.final_state = final_state;
        cp.norm_w = norm_w;
        cp.out = out;
        cp.c0 = c0;
        cp.c1 = c1;
        cp.slots = slots;
        cp.rec_chunks = rec_chunks;
        cp.state_rows = state_rows;
        if (pair) {
            int rc = smem_optin(reinterpret_cast<const void*>(gdn_chunk_pair_kernel), pair::SMEM_BYTES);
            if (rc != GDN_OK) return rc;
            cudaLaunchConfig_t cfg{};
            cfg.gridDim = dim3(2 * Vh, N);
            cfg.blockDim = dim3(pair::kThreads);
            cfg.dynamicSmemBytes = pair::SMEM_BYTES;
            cfg.stream = st;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            return cuda_status(cudaLaunchKernelEx(&cfg, gdn_chunk_pair_kernel, mV, mQ, mK, mZ, mO, cp));
        }
        int rc = smem_optin(reinterpret_cast<const void*>(gdn_chunk_kernel), chunk::SMEM_BYTES);
        if (rc != GDN_OK) return rc;
        dim3 grid(Vh, N);
        gdn_chunk_kernel<<<grid, chunk::kThreads, chunk::SMEM_BYTES, st>>>(mV, mQ, mK, mZ, mO, cp);
        return cuda_status(cudaGetLastError());
    }
};

int prefill_impl(const gdn_dims* d, const gdn_weights* w, int32_t N, const int32_t* cu_dev, int32_t uniform_T,
                 int32_t total, int64_t nchunks, int64_t nchunks_planned, const uint16_t* qkv, const uint16_t* z,
                 const uint16_t* a, const uint16_t* b, const float* init_state, const float* init_conv, uint16_t* out,
                 float* final_state, float* final_conv, void* workspace, size_t workspace_bytes, cudaStream_t stream,
                 bool may_overlap, const int32_t* slots_dev = nullptr, const FusedLoad* fused = nullptr,
                 const OutProjTail* op = nullptr, int32_t pool_rows = 0) {
    const int Kh = d->num_k_heads, Vh = d->num_v_heads;
    const int C = (2 * Kh + Vh) * 128;
    const size_t state_bytes = (size_t)N * Vh * 128 * 128 * 4;
    const size_t conv_bytes = (size_t)N * 3 * C * 4;
    SeqIndex seq{cu_dev, uniform_T, N};

    if (N == 0) return GDN_OK;
    if (total == 0) {
        // Nothing to run: states and histories pass through.
        if (final_state != nullptr && final_state != init_state) {
            cudaError_t e = init_state ? cudaMemcpyAsync(final_state, init_state, state_bytes, cudaMemcpyDeviceToDevice, stream)
                                       : cudaMemsetAsync(final_state, 0, state_bytes, stream);
            if (e != cudaSuccess) return GDN_ERR_CUDA;
        }
        if (final_conv != nullptr && final_conv != init_conv) {
            cudaError_t e = init_conv ? cudaMemcpyAsync(final_conv, init_conv, conv_bytes, cudaMemcpyDeviceToDevice, stream)
                                      : cudaMemsetAsync(final_conv, 0, conv_bytes, stream);
            if (e != cudaSuccess) return GDN_ERR_CUDA;
        }
        return GDN_OK;
    }

    const Workspace ws = plan_workspace(d, total, N, nchunks_planned);
    if (nchunks > nchunks_planned || nchunks > INT32_MAX / d->num_v_heads) return GDN_ERR_INVALID_ARG;
    if (workspace == nullptr || workspace_bytes < ws.bytes) return GDN_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDN_ERR_INVALID_ARG;
    uint8_t* wsb = static_cast<uint8_t*>(workspace);
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return GDN_ERR_CUDA;

    PrefillPlan P{};
    P.Kh = Kh;
    P.Vh = Vh;
    P.C = C;
    P.N = N;
    P.uniform_T = uniform_T;
    P.total = total;
    P.nsm = nsm;
    P.seq = seq;
    P.w = w;
    P.qkv = qkv;
    P.a = a;
    P.b = b;
    P.init_conv = init_conv;
    P.final_conv = final_conv;
    P.out = out;
    P.norm_w = w->norm_w;
    P.slots = slots_dev;
    P.fused = fused;
    P.Qs = reinterpret_cast<__half*>(wsb + ws.off_q);
    P.Ks = reinterpret_cast<__half*>(wsb + ws.off_k);
    P.Ql = reinterpret_cast<__half*>(wsb + ws.off_ql);
    P.Kl = reinterpret_cast<__half*>(wsb + ws.off_kl);
    P.Vs = reinterpret_cast<__half*>(wsb + ws.off_v);
    P.Gs = reinterpret_cast<float*>(wsb + ws.off_g);
    P.Bs = reinterpret_cast<float*>(wsb + ws.off_b);
    P.chunk_base = cu_dev ? reinterpret_cast<int*>(wsb + ws.off_cb) : nullptr;
    P.order = cu_dev ? P.chunk_base + N + 1 : nullptr;
    P.rec = wsb + ws.off_rec;
    P.rec_chunks = (int)nchunks_planned;
    P.state_rows = slots_dev != nullptr ? pool_rows : N;
    P.pair = use_pair(N, Vh, nsm);
    if (!make_map(&P.mK, P.Ks, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)Kh * 128, total, 64, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&P.mKl, P.Kl, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)Kh * 128, total, 64, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&P.mQl, P.Ql, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)Kh * 128, total, 64, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&P.mQ, P.Qs, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)Kh * 128, total, 64, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&P.mV, P.Vs, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (uint64_t)Vh * 128, total, 64, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&P.mZ, z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)Vh * 128, total, P.pair ? 64 : 128, 64,
                  P.pair ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&P.mO, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)Vh * 128, total, P.pair ? 64 : 128, 64,
                  P.pair ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE))
        return GDN_ERR_CUDA;

    // Overlapped schedule (dense rows that leave most SMs idle during the recurrence):
    // the load stage runs over all tokens first; then the rows' chunks are cut into S
    // segments and the WY records of segment s+1 run on the low-priority stream (a
    // persistent grid that leaves the recurrence its SMs) while the recurrence of
    // segment s runs on the high-priority one, each segment's recurrence starting from
    // the state the previous one left in final_state.
    const int chain_ctas = (P.pair ? 2 : 1) * N * Vh;
    SegPlan plan;
    if (may_overlap && cu_dev == nullptr && final_state != nullptr)
        plan = dense_plan(Kh, Vh, N, uniform_T, nsm, P.pair);
    const int S = plan.S;
    const int* cs = plan.cs;
    if (S > 1) {
        std::lock_guard<std::mutex> lock(g_side_mu);
        SideStreams* ss = nullptr;
        int st = side_streams(dev, &ss);
        if (st != GDN_OK) return st;
        if (cudaEventRecord(ss->fork, stream) != cudaSuccess || cudaStreamWaitEvent(ss->prod, ss->fork, 0) != cudaSuccess ||
            cudaStreamWaitEvent(ss->chain, ss->fork, 0) != cudaSuccess)
            return GDN_ERR_CUDA;
        if ((st = P.prep(0, total, ss->prod)) != GDN_OK) return st;
        for (int k = 0; k < S; ++k) {
            const int win = cs[k + 1] - cs[k];
            const int cap = k == 0 ? nsm : nsm - chain_ctas;  // leave the recurrence its SMs
            if ((st = P.wy_records((int64_t)N * win, cs[k], win, cap, ss->prod)) != GDN_OK) return st;
            if (cudaEventRecord(ss->seg[k], ss->prod) != cudaSuccess ||
                cudaStreamWaitEvent(ss->chain, ss->seg[k], 0) != cudaSuccess)
                return GDN_ERR_CUDA;
            if ((st = P.recurrence(cs[k], k + 1 < S ? cs[k + 1] : -1, k == 0 ? init_state : final_state, final_state,
                                   ss->chain)) != GDN_OK)
                return st;
            if (op != nullptr && cudaEventRecord(ss->rec[k], ss->chain) != cudaSuccess) return GDN_ERR_CUDA;
        }
        // out_proj on the lowest-priority stream: when the recurrence leaves at least half the
        // SMs, each segment's tokens as soon as that segment's recurrence has written them (it
        // takes the SMs the WY records leave); otherwise all tokens after the last segment (a
        // persistent GEMM grid between segments holds SMs the next recurrence launch needs:
        // one row on CTA pairs, 96 SMs, measured 0.86 ms per segment against 0.82 ms after)
        const bool per_segment = 2 * chain_ctas <= nsm;
        for (int k = per_segment ? 0 : S - 1; op != nullptr && k < S; ++k) {
            if (cudaStreamWaitEvent(ss->tail, ss->rec[k], 0) != cudaSuccess) return GDN_ERR_CUDA;
            const int64_t a0 = per_segment ? (int64_t)cs[k] * 64 : 0;
            const int64_t a1 = k + 1 < S ? (int64_t)cs[k + 1] * 64 : uniform_T;
            for (int n = 0; n < N; ++n)
                if ((st = out_proj_range(*op, out, Vh * 128, (int64_t)n * uniform_T + a0,
                                         (int64_t)n * uniform_T + (a1 < uniform_T ? a1 : uniform_T), ss->tail)) != GDN_OK)
                    return st;
        }
        // the final histories: after the load stage has read the old ones, off the path to the
        // first recurrence segment (beside the last one)
        if ((st = P.conv_out(ss->prod)) != GDN_OK) return st;
        if (cudaEventRecord(ss->prod_done, ss->prod) != cudaSuccess ||
            cudaEventRecord(ss->chain_done, ss->chain) != cudaSuccess ||
            cudaStreamWaitEvent(stream, ss->prod_done, 0) != cudaSuccess ||
            cudaStreamWaitEvent(stream, ss->chain_done, 0) != cudaSuccess)
            return GDN_ERR_CUDA;
        if (op != nullptr && (cudaEventRecord(ss->tail_done, ss->tail) != cudaSuccess ||
                              cudaStreamWaitEvent(stream, ss->tail_done, 0) != cudaSuccess))
            return GDN_ERR_CUDA;
        return GDN_OK;
    }

    // Plain schedule on the caller's stream.
    int st = P.prep(0, total, stream);  // 1. load stage: conv + silu, L2 norms, gates
    if (st != GDN_OK) return st;
    if ((st = P.conv_out(stream)) != GDN_OK) return st;  // 2. final history (after the load stage read it)
    if (P.chunk_base != nullptr) {                        // 3. first chunk of every packed row
        gdn_chunk_base_kernel<<<1, 1024, 0, stream>>>(cu_dev, N, P.chunk_base, P.order);
        if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    }
    if ((st = P.wy_records(nchunks, 0, 0, nsm, stream)) != GDN_OK) return st;  // 4. WY records, all chunks
    if ((st = P.recurrence(0, -1, init_state, final_state, stream)) != GDN_OK) return st;  // 5. recurrence + gated norm
    return op != nullptr ? out_proj_range(*op, out, Vh * 128, 0, total, stream) : GDN_OK;  // 6. out_proj
}

int check_io(int32_t total, const uint16_t* qkv, const uint16_t* z, const uint16_t* a, const uint16_t* b,
             const uint16_t* out, const float* init_state, const float* init_conv, const float* final_state,
             const float* final_conv) {
    if (total > 0) {
        if (!qkv || !z || !a || !b || !out) return GDN_ERR_INVALID_ARG;
        if (!aligned16(qkv) || !aligned16(z) || !aligned16(out)) return GDN_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(a) & 1u) || (reinterpret_cast<uintptr_t>(b) & 1u)) return GDN_ERR_INVALID_ARG;
    }
    const void* fs[4] = {init_state, init_conv, final_state, final_conv};
    for (const void* p : fs)
        if (p != nullptr && !aligned16(p)) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

// Scratch of gdn_prefill_noalloc: one fixed array per device, never freed.
// Host code must not pass g_noalloc_scratch itself to a kernel (on the host
// it names a stand-in, not the device address): its device address is looked
// up once per device below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[GDN_NOALLOC_SCRATCH_BYTES];

// The address is cached per CUDA context (by the driver's unique context id), so a
// context that replaced an earlier one on the same device (after cudaDeviceReset) gets
// its own lookup instead of a stale pointer.
std::mutex g_noalloc_mu;
struct NoallocEntry {
    unsigned long long ctx_id;
    void* addr;
};
std::vector<NoallocEntry> g_noalloc_addr;

using PfnCtxGetCurrent = CUresult (*)(CUcontext*);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long*);

void* driver_fn(const char* name) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion(name, &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return p;
}

// Unique id of the current context (0 if there is none or the driver cannot say).
unsigned long long current_ctx_id() {
    static PfnCtxGetCurrent get_cur = nullptr;
    static PfnCtxGetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        get_cur = reinterpret_cast<PfnCtxGetCurrent>(driver_fn("cuCtxGetCurrent"));
        get_id = reinterpret_cast<PfnCtxGetId>(driver_fn("cuCtxGetId"));
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_cur == nullptr || get_id == nullptr || get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of g_noalloc_scratch in the current context (resolved on first use there;
// cudaGetSymbolAddress also makes the device's primary context current if it was not).
int noalloc_scratch(void** out) {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    unsigned long long id = current_ctx_id();
    for (const NoallocEntry& e : g_noalloc_addr)
        if (id != 0 && e.ctx_id == id) {
            *out = e.addr;
            return GDN_OK;
        }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return GDN_ERR_CUDA;
    if (id == 0) id = current_ctx_id();
    if (id != 0) g_noalloc_addr.push_back(NoallocEntry{id, p});
    *out = p;
    return GDN_OK;
}

// Host check of a slot table: 0 <= slots[r] < pool_rows, no slot twice.
int check_slots(const int32_t* slots_host, int32_t rows, int32_t pool_rows) {
    if (slots_host == nullptr || pool_rows <= 0) return GDN_ERR_INVALID_ARG;
    std::vector<unsigned char> seen((size_t)pool_rows, 0);
    for (int32_t r = 0; r < rows; ++r) {
        const int32_t sl = slots_host[r];
        if (sl < 0 || sl >= pool_rows || seen[(size_t)sl]) return GDN_ERR_INVALID_ARG;
        seen[(size_t)sl] = 1;
    }
    return GDN_OK;
}

// The decode launch: rows batch rows, state / history rows through slots (or nullptr).
int decode_impl(const gdn_dims* dims, const gdn_weights* w, int32_t rows, const uint16_t* qkv, const uint16_t* z,
                const uint16_t* a, const uint16_t* b, float* state, float* conv, uint16_t* out, const int32_t* slots,
                int32_t ntok, void* stream, int32_t pool_rows) {
    int st = GDN_OK;
    if (!state || !conv || !aligned16(state) || !aligned16(conv)) return GDN_ERR_INVALID_ARG;
    if ((st = check_io(rows, qkv, z, a, b, out, nullptr, nullptr, nullptr, nullptr)) != GDN_OK) return st;
    if ((st = check_device()) != GDN_OK) return st;
    DecodeParams p{};
    p.Kh = dims->num_k_heads;
    p.Vh = dims->num_v_heads;
    p.C = (2 * p.Kh + p.Vh) * 128;
    p.rows = rows;
    p.qkv = qkv;
    p.z = z;
    p.a = a;
    p.b = b;
    p.conv_w = w->conv_w;
    p.A_log = w->A_log;
    p.dt_bias = w->dt_bias;
    p.norm_w = w->norm_w;
    p.state = state;
    p.conv = conv;
    p.out = out;
    p.slots = slots;
    p.pool_rows = pool_rows;
    p.ntok = ntok;
    const void* kernels[4] = {reinterpret_cast<const void*>(gdn_decode_kernel<1, false>),
                              reinterpret_cast<const void*>(gdn_decode_kernel<dec::kMaxTokens, false>),
                              reinterpret_cast<const void*>(gdn_decode_kernel<1, true>),
                              reinterpret_cast<const void*>(gdn_decode_kernel<dec::kMaxTokens, true>)};
    for (const void* k : kernels)
        if ((st = smem_optin(k, dec::kSmemLimit)) != GDN_OK) return st;
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return GDN_ERR_CUDA;
    // Work item = (row, q/k head) with its value heads, persistent CTAs walking the items.  A batch
    // small enough that one CTA per value head still fits in one wave splits each q/k group over a
    // cluster of Vh/Kh CTAs, one value head each (one item per CTA): 1 row 9.6 -> 6.3 us, 2 rows
    // 9.9 -> 6.5 us; with more than one wave the persistent grouping is faster.
    const int Gfull = p.Vh / p.Kh;
    const bool split = Gfull > 1 && rows * p.Kh * Gfull <= nsm;
    const int kmax = ntok == 1 ? 1 : dec::kMaxTokens;  // the kernel instantiation
    const dec::Plan dplan = dec::plan(split ? 1 : Gfull, ntok, dec::groups(kmax));
    if (dplan.stages < 2) return GDN_ERR_UNSUPPORTED;  // the group's inputs of ntok tokens leave no room
    p.nitems = rows * p.Kh * (split ? Gfull : 1);
    const int grid = split ? p.nitems : (p.nitems < nsm ? p.nitems : nsm);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(dec::threads(kmax));
    cfg.dynamicSmemBytes = dplan.smem_bytes;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = Gfull;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = split ? attr : nullptr;
    cfg.numAttrs = split ? 1 : 0;
    if (split)
        return cuda_status(ntok == 1 ? cudaLaunchKernelEx(&cfg, gdn_decode_kernel<1, true>, p)
                                     : cudaLaunchKernelEx(&cfg, gdn_decode_kernel<dec::kMaxTokens, true>, p));
    return cuda_status(ntok == 1 ? cudaLaunchKernelEx(&cfg, gdn_decode_kernel<1, false>, p)
                                 : cudaLaunchKernelEx(&cfg, gdn_decode_kernel<dec::kMaxTokens, false>, p));
}


// C = A W^T over bf16 A [M][K] and W [N][K], columns routed to the segments of gp.
int gemm_launch(const uint16_t* A, const uint16_t* W, GemmParams gp, cudaStream_t stream) {
    if (gp.M == 0 || gp.N == 0) return GDN_OK;
    if (gp.K <= 0 || gp.K % gemm::BK != 0) return GDN_ERR_UNSUPPORTED;
    if (!A || !W || !aligned16(A) || !aligned16(W)) return GDN_ERR_INVALID_ARG;
    for (int i = 0; i < gp.nseg; ++i)
        if (gp.seg[i].dst == nullptr || (reinterpret_cast<uintptr_t>(gp.seg[i].dst) & 1u)) return GDN_ERR_INVALID_ARG;
    int st = check_device();
    if (st != GDN_OK) return st;
    CUtensorMap mA, mW;
    if (!make_map(&mA, A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)gp.K, (uint64_t)gp.M, gemm::BK, gemm::BM,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mW, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)gp.K, (uint64_t)gp.N, gemm::BK, gemm::BN,
                  CU_TENSOR_MAP_SWIZZLE_128B))
        return GDN_ERR_CUDA;
    st = smem_optin(reinterpret_cast<const void*>(gdn_gemm_kernel<0>), gemm::SMEM_BYTES);
    if (st != GDN_OK) return st;
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return GDN_ERR_CUDA;
    const int64_t ntiles = (int64_t)((gp.M + gemm::BM - 1) / gemm::BM) * ((gp.N + gemm::BN - 1) / gemm::BN);
    const int grid = (int)(ntiles < nsm ? ntiles : nsm);
    gdn_gemm_kernel<0><<<grid, gemm::kThreads, gemm::SMEM_BYTES, stream>>>(mA, mW, gp, FusedPrep{});
    return cuda_status(cudaGetLastError());
}

// Workspace of gdn_prefill_hidden: the prefill workspace, then z, then either the
// rows' staged histories (fused load stage) or the unfused in_proj outputs.
struct HiddenLayout {
    bool fused;
    size_t off_z, off_conv, off_qkv, off_b, off_a, bytes;
};

// The fused load stage needs whole 256-column tiles of qkv and of z, and b and a in one tile.
bool fused_load_ok(const gdn_dims* d) {
    const int Kh = d->num_k_heads, Vh = d->num_v_heads;
    return (2 * Kh + Vh) % 2 == 0 && Vh % 2 == 0 && 2 * Vh <= gemm::BN;
}

// rows: N packed rows (or B dense rows) of `total` tokens in all; nchunks: the prefill's chunk plan
HiddenLayout hidden_layout(const gdn_dims* d, int32_t rows, int64_t total, int64_t nchunks) {
    HiddenLayout L{};
    const int Kh = d->num_k_heads, Vh = d->num_v_heads;
    const size_t C = (size_t)(2 * Kh + Vh) * 128;
    L.fused = fused_load_ok(d);
    L.off_z = plan_workspace(d, total, rows, nchunks).bytes;
    size_t o = L.off_z + align_up((size_t)total * Vh * 128 * 2);
    if (L.fused) {
        L.off_conv = o;
        o += align_up((size_t)rows * 3 * C * 4);
    } else {
        L.off_qkv = o;
        o += align_up((size_t)total * C * 2);
        L.off_b = o;
        o += align_up((size_t)total * Vh * 2);
        L.off_a = o;
        o += align_up((size_t)total * Vh * 2);
    }
    L.bytes = o;
    return L;
}

// The prefill from hidden states over dense rows (cu_dev == nullptr, uniform_T) or packed rows:
// the fused in_proj + load stage where the head counts allow, else in_proj then the prefill.
int prefill_hidden_impl(const gdn_dims* dims, const gdn_weights* w, int32_t N, const int32_t* cu_dev,
                        int32_t uniform_T, int32_t total, int64_t nch, int64_t nch_planned, int32_t hidden,
                        const uint16_t* x, const uint16_t* w_in, const float* init_state, const float* init_conv,
                        uint16_t* out, float* final_state, float* final_conv, void* workspace,
                        size_t workspace_bytes, void* stream) {
    int st = GDN_OK;
    if (hidden % gemm::BK != 0) return GDN_ERR_UNSUPPORTED;
    if (total > 0 && (!x || !w_in || !out || !aligned16(x) || !aligned16(w_in) || !aligned16(out)))
        return GDN_ERR_INVALID_ARG;
    const void* fs[4] = {init_state, init_conv, final_state, final_conv};
    for (const void* p : fs)
        if (p != nullptr && !aligned16(p)) return GDN_ERR_INVALID_ARG;
    if ((st = check_device()) != GDN_OK) return st;
    const HiddenLayout L = hidden_layout(dims, N, total, nch_planned);
    if (total > 0 && (workspace == nullptr || workspace_bytes < L.bytes)) return GDN_ERR_WORKSPACE;
    if (workspace != nullptr && !aligned16(workspace)) return GDN_ERR_INVALID_ARG;
    uint8_t* wsb = static_cast<uint8_t*>(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool dense = cu_dev == nullptr;
    uint16_t* z = total > 0 ? reinterpret_cast<uint16_t*>(wsb + L.off_z) : nullptr;
    if (total > 0 && L.fused) {
        FusedLoad fl{x, w_in, hidden, z, reinterpret_cast<float*>(wsb + L.off_conv)};
        return prefill_impl(dims, w, N, cu_dev, uniform_T, total, nch, nch_planned, nullptr, z, nullptr, nullptr,
                            init_state, init_conv, out, final_state, final_conv, workspace, L.off_z, s, dense,
                            nullptr, &fl);
    }
    // head counts the fused tiles do not cover: in_proj into the workspace, then the prefill over it
    uint16_t* qkv = total > 0 ? reinterpret_cast<uint16_t*>(wsb + L.off_qkv) : nullptr;
    uint16_t* bb = total > 0 ? reinterpret_cast<uint16_t*>(wsb + L.off_b) : nullptr;
    uint16_t* aa = total > 0 ? reinterpret_cast<uint16_t*>(wsb + L.off_a) : nullptr;
    if (total > 0 && (st = gdn_in_proj(dims, total, hidden, x, w_in, qkv, z, bb, aa, stream)) != GDN_OK) return st;
    return prefill_impl(dims, w, N, cu_dev, uniform_T, total, nch, nch_planned, qkv, z, aa, bb, init_state,
                        init_conv, out, final_state, final_conv, workspace, total > 0 ? L.off_z : 0, s, dense);
}

}  // namespace

extern "C" {

int gdn_in_proj(const gdn_dims* dims, int32_t T, int32_t hidden, const uint16_t* x, const uint16_t* w_in,
                uint16_t* qkv, uint16_t* z, uint16_t* b, uint16_t* a, void* stream) {
    NvtxRange nvtx_range("gdn_in_proj");
    int st = check_dims(dims);
    if (st != GDN_OK) return st;
    if (T < 0 || hidden <= 0) return GDN_ERR_INVALID_ARG;
    if (T == 0) return GDN_OK;
    const int Vh = dims->num_v_heads, D = dims->head_dim;
    const int C = (2 * dims->num_k_heads + Vh) * D;
    GemmParams gp{};
    gp.M = T;
    gp.N = C + Vh * D + 2 * Vh;
    gp.K = hidden;
    gp.nseg = 4;
    gp.seg[0] = GemmSegment{0, C, qkv};
    gp.seg[1] = GemmSegment{C, Vh * D, z};
    gp.seg[2] = GemmSegment{C + Vh * D, Vh, b};
    gp.seg[3] = GemmSegment{C + Vh * D + Vh, Vh, a};
    return gemm_launch(x, w_in, gp, static_cast<cudaStream_t>(stream));
}

int gdn_out_proj(const gdn_dims* dims, int32_t T, int32_t hidden, const uint16_t* y, const uint16_t* w_out,
                 uint16_t* out, void* stream) {
    NvtxRange nvtx_range("gdn_out_proj");
    int st = check_dims(dims);
    if (st != GDN_OK) return st;
    if (T < 0 || hidden <= 0) return GDN_ERR_INVALID_ARG;
    if (T == 0) return GDN_OK;
    GemmParams gp{};
    gp.M = T;
    gp.N = hidden;
    gp.K = dims->num_v_heads * dims->head_dim;
    gp.nseg = 1;
    gp.seg[0] = GemmSegment{0, hidden, out};
    return gemm_launch(y, w_out, gp, static_cast<cudaStream_t>(stream));
}


size_t gdn_prefill_hidden_workspace_size(const gdn_dims* dims, int32_t B, int32_t T) {
    if (check_dims(dims) != GDN_OK || B < 0 || T < 0) return 0;
    const int64_t total = (int64_t)B * T;
    if (total > INT32_MAX) return 0;
    return hidden_layout(dims, B, total, (int64_t)B * ((T + 63) / 64)).bytes;
}

int gdn_prefill_hidden(const gdn_dims* dims, const gdn_weights* w, int32_t B, int32_t T, int32_t hidden,
                       const uint16_t* x, const uint16_t* w_in, const float* init_state, const float* init_conv,
                       uint16_t* out, float* final_state, float* final_conv, void* workspace, size_t workspace_bytes,
                       void* stream) {
    NvtxRange nvtx_range("gdn_prefill_hidden");
    int st = check_dims(dims);
    if (st != GDN_OK) return st;
    if ((st = check_weights(w)) != GDN_OK) return st;
    if (B < 0 || T < 0 || B > 65535 || hidden <= 0) return GDN_ERR_INVALID_ARG;
    const int64_t total = (int64_t)B * T;
    if (total > INT32_MAX) return GDN_ERR_INVALID_ARG;
    const int64_t nch = (int64_t)B * ((T + 63) / 64);
    return prefill_hidden_impl(dims, w, B, nullptr, T, (int32_t)total, nch, nch, hidden, x, w_in, init_state,
                               init_conv, out, final_state, final_conv, workspace, workspace_bytes, stream);
}

size_t gdn_prefill_hidden_varlen_workspace_size(const gdn_dims* dims, int32_t N, int32_t total_T) {
    if (check_dims(dims) != GDN_OK || N < 0 || total_T < 0) return 0;
    return hidden_layout(dims, N, total_T, chunk_bound(N, total_T)).bytes;
}

int gdn_prefill_hidden_varlen(const gdn_dims* dims, const gdn_weights* w, int32_t N, const int32_t* cu_host,
                              const int32_t* cu_dev, int32_t total_T, int32_t hidden, const uint16_t* x,
                              const uint16_t* w_in, const float* init_state, const float* init_conv, uint16_t* out,
                              float* final_state, float* final_conv, void* workspace, size_t workspace_bytes,
                              void* stream) {
    NvtxRange nvtx_range("gdn_prefill_hidden_varlen");
    int st = check_dims(dims);
    if (st != GDN_OK) return st;
    if ((st = check_weights(w)) != GDN_OK) return st;
    if (N < 0 || N > 65535 || total_T < 0 || hidden <= 0) return GDN_ERR_INVALID_ARG;
    if (cu_host == nullptr || (N > 0 && cu_dev == nullptr)) return GDN_ERR_INVALID_ARG;
    if (cu_host[0] != 0 || cu_host[N] != total_T) return GDN_ERR_INVALID_ARG;
    for (int32_t i = 0; i < N; ++i)
        if (cu_host[i + 1] < cu_host[i]) return GDN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(cu_dev) & 3u) != 0) return GDN_ERR_INVALID_ARG;
    int64_t nch = 0;
    for (int32_t i = 0; i < N; ++i) nch += (cu_host[i + 1] - cu_host[i] + 63) / 64;
    return prefill_hidden_impl(dims, w, N, cu_dev, 0, total_T, nch, chunk_bound(N, total_T), hidden, x, w_in,
                               init_state, init_conv, out, final_state, final_conv, workspace, workspace_bytes,
                               stream);
}

// The schedule of a dense prefill on a device with nsm SMs (arguments already checked).
void schedule_for(const gdn_dims* dims, int32_t B, int32_t T, int32_t from_hidden, int nsm, int32_t* segments,
                  int32_t* launches) {
    const bool fused = from_hidden != 0 && fused_load_ok(dims);
    const SegPlan pl =
        dense_plan(dims->num_k_heads, dims->num_v_heads, B, T, nsm, use_pair(B, dims->num_v_heads, nsm));
    *segments = pl.S;
    *launches = plan_launches(pl) + (from_hidden != 0 && !fused ? 1 : 0);  // + the unfused in_proj
}

int schedule_args(const gdn_dims* dims, int32_t B, int32_t T, int32_t* segments, int32_t* launches) {
    int st = check_dims(dims);
    if (st != GDN_OK) return st;
    if (B < 0 || T < 0 || B > 65535 || (int64_t)B * T > INT32_MAX || !segments || !launches)
        return GDN_ERR_INVALID_ARG;
    *segments = 0;
    *launches = 0;
    return GDN_OK;
}

int gdn_prefill_schedule(const gdn_dims* dims, int32_t B, int32_t T, int32_t from_hidden, int32_t* segments,
                         int32_t* launches) {
    int st = schedule_args(dims, B, T, segments, launches);
    if (st != GDN_OK || B == 0 || T == 0) return st;
    if ((st = check_device()) != GDN_OK) return st;
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return GDN_ERR_CUDA;
    schedule_for(dims, B, T, from_hidden, nsm, segments, launches);
    return GDN_OK;
}

int gdn_prefill_schedule_nsm(const gdn_dims* dims, int32_t B, int32_t T, int32_t from_hidden, int32_t nsm,
                             int32_t* segments, int32_t* launches) {
    int st = schedule_args(dims, B, T, segments, launches);
    if (st != GDN_OK) return st;
    if (nsm < 1) return GDN_ERR_INVALID_ARG;
    if (B == 0 || T == 0) return GDN_OK;
    schedule_for(dims, B, T, from_hidden, nsm, segments, launches);
    return GDN_OK;
}

size_t gdn_prefill_workspace_size(const gdn_dims* dims, int32_t B, int32_t T) {
    if (check_dims(dims) != GDN_OK || B < 0 || T < 0) return 0;
    const int64_t total = (int64_t)B * T;
    if (total > INT32_MAX) return 0;
    return plan_workspace(dims, total, B, (int64_t)B * ((T + 63) / 64)).bytes;
}

size_t gdn_prefill_out_workspace_size(const gdn_dims* dims, int32_t B, int32_t T) {
    if (check_dims(dims) != GDN_OK || B < 0 || T < 0) return 0;
    const int64_t total = (int64_t)B * T;
    if (total > INT32_MAX) return 0;
    return plan_workspace(dims, total, B, (int64_t)B * ((T + 63) / 64)).bytes +
           align_up((size_t)total * dims->num_v_heads * 128 * 2);
}

int gdn_prefill_out(const gdn_dims* dims, const gdn_weights* w, int32_t B, int32_t T, int32_t hidden,
                    const uint16_t* qkv, const uint16_t* z, const uint16_t* a, const uint16_t* b,
                    const float* init_state, const float* init_conv, const uint16_t* w_out, uint16_t* out,
                    float* final_state, float* final_conv, void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("gdn_prefill_out");
    int st = check_dims(dims);
    if (st != GDN_OK) return st;
    if ((st = check_weights(w)) != GDN_OK) return st;
    if (B < 0 || T < 0 || B > 65535 || hidden <= 0) return GDN_ERR_INVALID_ARG;
    if (hidden % 8 != 0) return GDN_ERR_UNSUPPORTED;
    const int64_t total = (int64_t)B * T;
    if (total > INT32_MAX) return GDN_ERR_INVALID_ARG;
    if ((st = check_io((int32_t)total, qkv, z, a, b, out, init_state, init_conv, final_state, final_conv)) != GDN_OK)
        return st;
    if (total > 0 && (w_out == nullptr || !aligned16(w_out))) return GDN_ERR_INVALID_ARG;
    if ((st = check_device()) != GDN_OK) return st;
    const int64_t nch = (int64_t)B * ((T + 63) / 64);
    const size_t ws_mixer = plan_workspace(dims, total, B, nch).bytes;
    if (total > 0 && (workspace == nullptr || workspace_bytes < gdn_prefill_out_workspace_size(dims, B, T)))
        return GDN_ERR_WORKSPACE;
    uint16_t* y = total > 0 ? reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(workspace) + ws_mixer) : nullptr;
    const OutProjTail op{w_out, hidden, out};
    return prefill_impl(dims, w, B, nullptr, T, (int32_t)total, nch, nch, qkv, z, a, b, init_state, init_conv, y,
                        final_state, final_conv, workspace, ws_mixer, static_cast<cudaStream_t>(stream), true, nullptr,
                        nullptr, &op);
}

size_t gdn_prefill_varlen_workspace_size(const gdn_dims* dims, int32_t N, int32_t total_T) {
    if (check_dims(dims) != GDN_OK || N < 0 || total_T < 0) return 0;
    return plan_workspace(dims, total_T, N, chunk_bound(N, total_T)).bytes;
}

int gdn_prefill(const gdn_dims* dims, const gdn_weights* w, int32_t B, int32_t T, const uint16_t* qkv,
                const uint16_t* z, const uint16_t* a, const uint16_t* b, const float* init_state,
                const float* init_conv, uint16_t* out, float* final_state, float* final_conv, void* workspace,
                size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("gdn_prefill");
    int st = check_dims(dims);
    if (st != GDN_OK) return st;
    if ((st = check_weights(w)) != GDN_OK) return st;
    if (B < 0 || T < 0 || B > 65535) return GDN_ERR_INVALID_ARG;
    const int64_t total = (int64_t)B * T;
    if (total > INT32_MAX) return GDN_ERR_INVALID_ARG;
    if ((st = check_io((int32_t)total, qkv, z, a, b, out, init_state, init_conv, final_state, final_conv)) != GDN_OK)
        return st;
    if ((st = check_device()) != GDN_OK) return st;
    const int64_t nch = (int64_t)B * ((T + 63) / 64);
    return prefill_impl(dims, w, B, nullptr, T, (int32_t)total, nch, nch, qkv, z, a, b, init_state, init_conv, out,
                        final_state, final_conv, workspace, workspace_bytes, static_cast<cudaStream_t>(stream), true);
}

int gdn_prefill_varlen(const gdn_dims* dims, const gdn_weights* w, int32_t N, const int32_t* cu_host,
                       const int32_t* cu_dev, int32_t total_T, const uint16_t* qkv, const uint16_t* z,
                       const uint16_t* a, const uint16_t* b, const float* init_state, const float* init_conv,
                       uint16_t* out, float* final_state, float* final_conv, void* workspace, size_t workspace_bytes,
                       void* stream) {
    NvtxRange nvtx_range("gdn_prefill_varlen");
    int st = check_dims(dims);
    if (st != GDN_OK) return st;
    if ((st = check_weights(w)) != GDN_OK) return st;
    if (N < 0 || N > 65535 || total_T < 0) return GDN_ERR_INVALID_ARG;
    if (cu_host == nullptr || (N > 0 && cu_dev == nullptr)) return GDN_ERR_INVALID_ARG;
    if (cu_host[0] != 0 || cu_host[N] != total_T) return GDN_ERR_INVALID_ARG;
    for (int32_t i = 0; i < N; ++i)
        if (cu_host[i + 1] < cu_host[i]) return GDN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(cu_dev) & 3u) != 0) return GDN_ERR_INVALID_ARG;
    if ((st = check_io(total_T, qkv, z, a, b, out, init_state, init_conv, final_state, final_conv)) != GDN_OK)
        return st;
    if ((st = check_device()) != GDN_OK) return st;
    int64_t nch = 0;
    for (int32_t i = 0; i < N; ++i) nch += (cu_host[i + 1] - cu_host[i] + 63) / 64;
    return prefill_impl(dims, w, N, cu_dev, 0, total_T, nch, chunk_bound(N, total_T), qkv, z, a, b, init_state,
                        init_conv, out, final_state, final_conv, workspace, workspace_bytes,
                        static_cast<cudaStream_t>(stream), false);
}

int gdn_decode(const gdn_dims* dims, const gdn_weights* w, int32_t rows, const uint16_t* qkv, const uint16_t* z,
               const uint16_t* a, const uint16_t* b, float* state, float* conv, uint16_t* out, void* stream) {
    NvtxRange nvtx_range("gdn_decode");
    int st = check_dims(dims);
    if (st != GDN_OK) return st;
    if ((st = check_weights(w)) != GDN_OK) return st;
    if (rows < 0 || rows > 65535) return GDN_ERR_INVALID_ARG;
    if (rows == 0) return GDN_OK;
    return decode_impl(dims, w, rows, qkv, z, a, b, state, conv, out, nullptr, 1, stream, rows);
}

int gdn_decode_multi(const gdn_dims* dims, const gdn_weights* w, int32_t rows, int32_t ntok, const uint16_t* qkv,
                     const uint16_t* z, const uint16_t* a, const uint16_t* b, float* state, float* conv, uint16_t* out,
                     void* stream) {
    NvtxRange nvtx_range("gdn_decode_multi");
    int st = check_dims(dims);
    if (st != GDN_OK) return st;
    if ((st = check_weights(w)) != GDN_OK) return st;
    if (rows < 0 || rows > 65535 || ntok < 1) return GDN_ERR_INVALID_ARG;
    if (ntok > dec::kMaxTokens) return GDN_ERR_UNSUPPORTED;
    if (rows == 0) return GDN_OK;
    return decode_impl(dims, w, rows, qkv, z, a, b, state, conv, out, nullptr, ntok, stream, rows);
}


int gdn_decode_slots(const gdn_dims* dims, const gdn_weights* w, int32_t rows, const int32_t* slots_host,
                     const int32_t* slots_dev, int32_t pool_rows, const uint16_t* qkv, const uint16_t* z,
                     const uint16_t* a, const uint16_t* b, float* state_pool, float* conv_pool, uint16_t* out,
                     void* stream) {
    NvtxRange nvtx_range("gdn_decode_slots");
    int st = check_dims(dims);
    if (st != GDN_OK) return st;
    if ((st = check_weights(w)) != GDN_OK) return st;
    if (rows < 0 || rows > 65535) return GDN_ERR_INVALID_ARG;
    if (rows == 0) return GDN_OK;
    if ((st = check_slots(slots_host, rows, pool_rows)) != GDN_OK) return st;
    if (slots_dev == nullptr || (reinterpret_cast<uintptr_t>(slots_dev) & 3u)) return GDN_ERR_INVALID_ARG;
    return decode_impl(dims, w, rows, qkv, z, a, b, state_pool, conv_pool, out, slots_dev, 1, stream, pool_rows);
}

int gdn_prefill_varlen_slots(const gdn_dims* dims, const gdn_weights* w, int32_t N, const int32_t* cu_host,
                             const int32_t* cu_dev, int32_t total_T, const int32_t* slots_host,
                             const int32_t* slots_dev, int32_t pool_rows, const uint16_t* qkv, const uint16_t* z,
                             const uint16_t* a, const uint16_t* b, float* state_pool, float* conv_pool,
                             uint16_t* out, void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("gdn_prefill_varlen_slots");
    int st = check_dims(dims);
    if (st != GDN_OK) return st;
    if ((st = check_weights(w)) != GDN_OK) return st;
    if (N < 0 || N > 65535 || total_T < 0) return GDN_ERR_INVALID_ARG;
    if (cu_host == nullptr || (N > 0 && cu_dev == nullptr)) return GDN_ERR_INVALID_ARG;
    if (cu_host[0] != 0 || cu_host[N] != total_T) return GDN_ERR_INVALID_ARG;
    for (int32_t i = 0; i < N; ++i)
        if (cu_host[i + 1] < cu_host[i]) return GDN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(cu_dev) & 3u) != 0) return GDN_ERR_INVALID_ARG;
    if (N == 0) return GDN_OK;
    if ((st = check_slots(slots_host, N, pool_rows)) != GDN_OK) return st;
    if (slots_dev == nullptr || (reinterpret_cast<uintptr_t>(slots_dev) & 3u)) return GDN_ERR_INVALID_ARG;
    if (state_pool == nullptr || conv_pool == nullptr) return GDN_ERR_INVALID_ARG;
    if ((st = check_io(total_T, qkv, z, a, b, out, state_pool, conv_pool, state_pool, conv_pool)) != GDN_OK)
        return st;
    if ((st = check_device()) != GDN_OK) return st;
    if (total_T == 0) return GDN_OK;  // the pool rows stay as they are
    int64_t nch = 0;
    for (int32_t i = 0; i < N; ++i) nch += (cu_host[i + 1] - cu_host[i] + 63) / 64;
    return prefill_impl(dims, w, N, cu_dev, 0, total_T, nch, chunk_bound(N, total_T), qkv, z, a, b, state_pool,
                        conv_pool, out, state_pool, conv_pool, workspace, workspace_bytes,
                        static_cast<cudaStream_t>(stream), false, slots_dev, nullptr, nullptr, pool_rows);
}

int gdn_prefill_noalloc(const gdn_dims* dims, const gdn_weights* w, int32_t B, int32_t T, const uint16_t* qkv,
                        const uint16_t* z, const uint16_t* a, const uint16_t* b, const float* init_state,
                        const float* init_conv, uint16_t* out, float* final_state, float* final_conv, void* stream) {
    NvtxRange nvtx_range("gdn_prefill_noalloc");
    int st = check_dims(dims);
    if (st != GDN_OK) return st;
    if ((st = check_weights(w)) != GDN_OK) return st;
    if (B < 0 || T < 0 || B > 65535) return GDN_ERR_INVALID_ARG;
    const int64_t total = (int64_t)B * T;
    if (total > INT32_MAX) return GDN_ERR_INVALID_ARG;
    if ((st = check_io((int32_t)total, qkv, z, a, b, out, init_state, init_conv, final_state, final_conv)) != GDN_OK)
        return st;
    const int64_t nch = (int64_t)B * ((T + 63) / 64);
    if (plan_workspace(dims, total, B, nch).bytes > (size_t)GDN_NOALLOC_SCRATCH_BYTES) return GDN_ERR_WORKSPACE;
    if ((st = check_device()) != GDN_OK) return st;
    void* scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != GDN_OK) return st;
    return prefill_impl(dims, w, B, nullptr, T, (int32_t)total, nch, nch, qkv, z, a, b, init_state, init_conv, out,
                        final_state, final_conv, scratch, (size_t)GDN_NOALLOC_SCRATCH_BYTES,
                        static_cast<cudaStream_t>(stream), false);
}

int gdn_set_decode_wait_limit(uint64_t ns) {
    if (cudaDeviceSynchronize() != cudaSuccess) return GDN_ERR_CUDA;
    const unsigned long long v = ns;
    if (cudaMemcpyToSymbol(gdn::g_decode_wait_limit_ns, &v, sizeof(v)) != cudaSuccess) return GDN_ERR_CUDA;
    return cudaDeviceSynchronize() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

int gdn_test_decode_stop_copies_at(int32_t unit) {
    if (unit < -1) return GDN_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return GDN_ERR_CUDA;
    const int v = unit;
    if (cudaMemcpyToSymbol(gdn::g_decode_stop_copies_at, &v, sizeof(v)) != cudaSuccess) return GDN_ERR_CUDA;
    return cudaDeviceSynchronize() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

int gdn_last_device_error(void) {
    int v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return GDN_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, gdn::g_device_error, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(gdn::g_device_error, &zero, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
    return v;
}

const char* gdn_status_string(int status) {
    switch (status) {
        case GDN_OK: return "ok";
        case GDN_ERR_INVALID_ARG: return "invalid argument";
        case GDN_ERR_UNSUPPORTED: return "unsupported dimensions or device";
        case GDN_ERR_CUDA: return "CUDA error";
        case GDN_ERR_WORKSPACE: return "workspace missing or too small";
        case GDN_ERR_TIMEOUT: return "bounded device wait expired";
        default: return "unknown status";
    }
}

int gdn_version(void) { return 100; }

}  // extern "C"
