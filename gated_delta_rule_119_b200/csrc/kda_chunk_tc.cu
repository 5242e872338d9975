// Chunked KDA prefill on the sm_100a tensor cores (bf16 q/k/v, dk = dv = 128, C = 64).
//
// Chunk algebra ("22,580" §6.3 WY/UT form with the per-channel cumulative decay of
// its §08/§9.1).  Inside a chunk every decay factor is a product of alphas over the
// steps strictly after a write up to its read, D[r][i] = prod_{i<s<=r} alpha_s:
//
//   A[r][i]  = beta_r sum_c k_rc k_ic D_ric  (i < r),   P[r][i] = s sum_c q_rc k_ic D_ric  (i <= r)
//   T'       = (I + A)^{-1} Diag(beta),  W = T' (k gamma),  gamma_r = prod_{s<=r} alpha_s
//   u        = T' v - W S
//   o        = (s q gamma) S + P u  =  (s q gamma - P W) S + (P T') v
//   S       <- Diag(gamma_last) S + (k kappa)^T u,   kappa_i = prod_{s>i} alpha_s
//
// so one tensor-core accumulation gives u (rows 0-63) and o (rows 64-127):
//   [u; o] = [T'; P T'] v + [-W; s q gamma - P W] S.
//
// Two kernels.  The intra-chunk kernel works on every (chunk, head) independently --
// nothing in it depends on the state -- and writes the chunk's tensor-core operands
// [T'; P T'], [-W; s q gamma - P W], the update operand and gamma_last into one
// workspace slot, already in the shared-memory image the tensor core reads.  The scan
// kernel walks each (sequence, head, 64-column slice of d_v) chunk by chunk with
// specialised warps: one fetches the next slot (bulk copy) and v tile (TMA) while the
// current chunk runs, one issues the tensor-core products, eight move the state, u and o
// through tensor memory, and one stores o (TMA).
//
// Intra-chunk kernel, per (chunk, head), instantiated per gate form:
//  IN  one thread loads the chunk's gate tile (log_alpha fp32, or the fused gate's f), k and q
//      by TMA into shared memory that later phases reuse (a scalar gate is read like beta);
//      with unit-length keys / queries asked for, the rows' norms are summed from the tiles.
//  E2  one thread per (2 channels, 16-row block): log_alpha (computed from f for the fused
//      gate), alpha = exp(log_alpha), block-local running products, and from them k gamma,
//      s q gamma (tensor-core operand) and the update operand.
//  AP  Fast path -- every channel's decay over the chunk within e^-80: A and P from one
//      tcgen05 product [k gamma; s q gamma] (k e^-g)^T, and the update operand is
//      k e^-g (the state update becomes Diag(gamma_last)(S + (k e^-g)^T u), its decay
//      applied when the state is next read).  Block path otherwise: 16 x 16 blocks of A
//      and P with block-local decay references rescaled into [e^-70, e^70] (warp MMAs),
//      an exact per-channel path for blocks whose spread exceeds that range, and the
//      update operand k kappa.
//  T   T = (I + A)^{-1}: 16 x 16 diagonal blocks by substitution in fp32, the rest with
//      tf32 warp MMAs; [T'; P T'] = [I; P] T' and
//      [-W; s q gamma - P W] = [0; s q gamma] - [T'; P T'] (k gamma) on tcgen05.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdio.h>
#include <string.h>

#include <atomic>

#include "kda_common.cuh"
#include "kda_tc_util.cuh"

__device__ unsigned int g_kda_device_status = 0;

namespace {
using namespace kda_tc;

constexpr int CH = 64, DK = 128, DV = 128;
constexpr int DVT = 64;                 // d_v columns per scan CTA
constexpr int NTILE = DV / DVT;         // scan CTAs per (sequence, head)
constexpr int NTHR = 256;
constexpr int LF = 68;                  // row pitch (fp32) of the 64 x 64 matrices
constexpr float kSpreadLimit = 140.f;   // -sum log_alpha over 16 rows beyond which a block is exact-path
constexpr float kChunkSpreadLimit = 80.f;   // -sum log_alpha over a chunk for the fast path
constexpr long long kWaitCycles = 4000000000LL;   // about 2 s at B200 clocks

// Workspace slot of one (chunk, head), the shared-memory image of the scan's operands.
constexpr uint32_t SLOT_TP = 0;         // [T'; P T']: 128 lines (K-major A)
constexpr uint32_t SLOT_A2 = 16384;     // [-W; s q gamma - P W]: 2 x 128 lines (K-major A)
constexpr uint32_t SLOT_KC = 49152;     // update operand: 2 x 64 lines (MN-major A)
constexpr uint32_t SLOT_GC = 65536;     // gamma_last [128] fp32
constexpr uint32_t SLOT_FLAG = 66048;   // 1 = fast path (decay deferred), 0 = block path
constexpr uint32_t SLOT_BYTES = 66560;

// Intra-chunk kernel shared memory (bytes from a 1024-aligned base); two CTAs per SM.
constexpr uint32_t I_KQ = 0;            // [k gamma; s q gamma]: 2 x 128 lines
constexpr uint32_t I_KC = 32768;        // k e^-g (fast-path B operand of A, P) or the block
                                        //   path's right k factor, then [I; P]
constexpr uint32_t I_AM = 49152;        // the block path's left k factor, then A [64][LF] fp32
constexpr uint32_t I_TM = 66560;        // T [64][LF] fp32; before it, the block path's scale
                                        //   table [10][128] and exact-path P [4][16][16]
constexpr uint32_t I_SC = I_TM, I_CP = I_TM + 5120, I_CA = I_TM + 9216;   // I_CA: exact-path A [4][16][16]
constexpr uint32_t I_TP = 83968;        // q (then the block path's left s q factor), then [T'; P T']
constexpr uint32_t I_BETA = 100352;     // [64]
constexpr uint32_t I_GC = I_BETA + 256; // [128]
constexpr uint32_t I_BS = I_GC + 512;   // [4][128] sum of log_alpha per 16-row block
constexpr uint32_t I_BT = I_BS + 2048;  // [4][128] product of alpha per block
constexpr uint32_t I_XT = I_BT + 2048;  // [6][128] forward-substitution scratch
constexpr uint32_t I_RK = I_XT + 3072;  // [64] 1 / ||k_r|| (unit-length keys), else unused
constexpr uint32_t I_RQ = I_RK + 256;   // [64] 1 / ||q_r|| (unit-length queries), else unused
constexpr uint32_t I_LA = I_RQ + 256;   // [64] the scalar gate's log alpha per row
constexpr uint32_t I_END = I_LA + 256;
constexpr size_t kIntraSmem = I_END + 1024;
static_assert(I_TP % 1024 == 0 && I_KC % 1024 == 0, "tile alignment");
static_assert(I_CA + 4096 <= I_TP, "block-path scratch inside T");
static_assert(I_AM + 32768 <= I_TP, "[-W; s q gamma - P W] staged in the space of A and T");
static_assert(2 * (kIntraSmem + 1024) <= 233472, "two intra CTAs per SM");

// Scan kernel shared memory: two stages of {slot image, v slice}, the bf16 state copy, two o
// staging tiles.
constexpr uint32_t S_STAGE = 74752;     // SLOT_BYTES + 8192 (v slice), 1024-aligned
constexpr uint32_t S_V = SLOT_BYTES;    // v slice of the chunk, then u: 64 lines (MN-major B)
constexpr uint32_t S_S = 2 * S_STAGE;   // bf16 state copy: 128 lines (MN-major B)
constexpr uint32_t S_O = S_S + 16384;   // o of a chunk's d_v tile, [64 tokens][64] bf16 (one TMA box)
constexpr uint32_t S_END = S_O + 2 * 8192;
constexpr size_t kScanSmem = S_END + 1024;
static_assert(S_STAGE % 1024 == 0 && S_V % 1024 == 0 && S_S % 1024 == 0 && S_O % 1024 == 0, "tile alignment");
static_assert(kScanSmem <= 232448, "shared memory budget");

__constant__ int kPairA[10] = {0, 1, 1, 2, 2, 2, 3, 3, 3, 3};
__constant__ int kPairB[10] = {0, 0, 1, 0, 1, 2, 0, 1, 2, 3};

__device__ __forceinline__ uint4 pack8(const float *v) {
    uint4 pk;
    pk.x = pack_bf16(v[0], v[1]);
    pk.y = pack_bf16(v[2], v[3]);
    pk.z = pack_bf16(v[4], v[5]);
    pk.w = pack_bf16(v[6], v[7]);
    return pk;
}

// x scaled by the row's unit-length factor (NORM) or unchanged.
template <bool NORM>
__device__ __forceinline__ float2 row_scaled(float2 x, const float *f, int r) {
    if (!NORM) return x;
    const float s = f[r];
    return make_float2(x.x * s, x.y * s);
}

// Byte offset of element (r, c) of a [64][128] bf16 tile stored as two 64-column halves of
// 128-byte rows, the 16-byte chunks of row r XOR-swizzled by r & 7 (the layout a TMA load with
// 128-byte swizzle writes): conflict-free both for a warp reading 32 consecutive channels of one
// row and for the warp-MMA fragment loads (8 rows x 4 column pairs).
__device__ __forceinline__ uint32_t rm_sw(int r, int c) {
    return (uint32_t)((c >> 6) * 8192 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1));
}

// Varlen bookkeeping in the workspace head: base[n] = sum_{m<n} ceil(len_m / 64) (the slot
// offsets), and order[0..N) = the sequences by decreasing length (ties by index), so the scan
// starts its longest chains first.  Up to kSortMax sequences are ranked; beyond that the order
// is the identity.
// Well-formed offsets need at most ceil(T_total / 64) + N slots, the workspace's size.  Offsets
// that are not non-decreasing can make clamped sequences overlap and ask for more; the running
// sum is therefore capped at max_slots, so a sequence gets min(its chunks, the slots left), and
// the scan walks only base[n + 1] - base[n] chunks of sequence n: no slot outside the workspace
// is ever written or read (the results of such a call are unspecified).
constexpr int kSortMax = 256;

__global__ void __launch_bounds__(kSortMax) kda_chunk_slots_kernel(const int32_t *cu_seqlens, int N,
                                                                    int64_t T_total, int64_t max_slots,
                                                                    int32_t *base, int32_t *order) {
    if (threadIdx.x == 0) {
        int64_t acc = 0;
        for (int n = 0; n < N; ++n) {
            int64_t t0, t1;
            kda::seq_bounds(cu_seqlens, n, 0, T_total, t0, t1);
            base[n] = (int32_t)acc;
            const int64_t want = (t1 - t0 + CH - 1) / CH;
            acc += want < max_slots - acc ? want : max_slots - acc;
        }
        base[N] = (int32_t)acc;
    }
    if (N > kSortMax) {
        for (int n = threadIdx.x; n < N; n += blockDim.x) order[n] = n;
        return;
    }
    __shared__ int64_t len[kSortMax];
    const int t = threadIdx.x;
    if (t < N) {
        int64_t t0, t1;
        kda::seq_bounds(cu_seqlens, t, 0, T_total, t0, t1);
        len[t] = t1 - t0;
    }
    __syncthreads();
    if (t < N) {
        int rank = 0;
        for (int m = 0; m < N; ++m) rank += (len[m] > len[t] || (len[m] == len[t] && m < t)) ? 1 : 0;
        order[rank] = t;
    }
}

// Exact diagonal-block contributions of the channels whose decay over a 16-row block is too
// strong for the rescaled factors (-sum log_alpha over the block > kSpreadLimit): running
// products of alpha, inputs re-read from memory.  Thread t takes block t / 64, column
// i = (t / 4) % 16, the row half rh = (t / 2) % 2 (rows 8 rh .. 8 rh + 7 of the block) and the
// channel half t % 2: over its flagged channels, in channel order, it carries the running
// product D_Ri from row i down its rows; then the two channel halves of (block, i, rh) --
// adjacent lanes -- are added.  Writes sCA[blk][R][i] = sum beta_R k_R k_i D_Ri (i < R) and
// sCP[blk][R][i] = sum s q_R k_i D_Ri (i <= R) for the rows of the chunk, the same on every run.
// Called by all NTHR threads of the CTA.  With NORM, k and q are scaled by the rows' unit-length
// factors sRk, sRq.
template <int GATE, bool NORM>
__device__ __noinline__ void exact_diag_blocks(const KdaChunkArgs &a, int64_t c0, int nr, int h, const float *sBS,
                                               const float *sBeta, const float *sRk, const float *sRq,
                                               float *sCA, float *sCP) {
    const int H = a.H;
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(a.q);
    const __nv_bfloat16 *kg = static_cast<const __nv_bfloat16 *>(a.k);
    const int t = threadIdx.x, chh = t & 1, rh = (t >> 1) & 1, i = (t >> 2) & 15, blk = t >> 6;
    const int I = 16 * blk + i;
    float sa[8], sp[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) sa[r] = sp[r] = 0.f;
    if (I < nr && 8 * rh + 7 >= i) {
        for (int cc = 0; cc < DK / 2; ++cc) {
            const int ch = (DK / 2) * chh + cc;
            if (!(sBS[blk * 128 + ch] < -kSpreadLimit)) continue;
            float ki = __bfloat162float(kg[((size_t)(c0 + I) * H + h) * DK + ch]);
            if (NORM) ki *= sRk[I];
            float f = 1.f;
            for (int R = i + 1; R < 8 * rh && 16 * blk + R < nr; ++R)   // rows before this half
                f *= __expf(kda::gate_log_alpha<__nv_bfloat16>(GATE, a.gate, a.A_log, a.dt_bias,
                                                                (size_t)(c0 + 16 * blk + R) * H + h, h, ch, DK));
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int R = 8 * rh + r, Rg = 16 * blk + R;
                if (R >= i && Rg < nr) {
                    const size_t th = (size_t)(c0 + Rg) * H + h, off = th * DK + ch;
                    if (R > i)
                        f *= __expf(kda::gate_log_alpha<__nv_bfloat16>(GATE, a.gate, a.A_log, a.dt_bias, th, h, ch, DK));
                    const float kd = ki * f;
                    const float kr = __bfloat162float(kg[off]) * (NORM ? sRk[Rg] : 1.f);
                    const float qr = __bfloat162float(qg[off]) * (NORM ? sRq[Rg] : 1.f);
                    if (R > i) sa[r] += sBeta[Rg] * kr * kd;
                    sp[r] += a.scale * qr * kd;
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        sa[r] += __shfl_xor_sync(0xffffffffu, sa[r], 1);
        sp[r] += __shfl_xor_sync(0xffffffffu, sp[r], 1);
    }
    if (chh == 0) {
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            sCA[blk * 256 + (8 * rh + r) * 16 + i] = sa[r];
            sCP[blk * 256 + (8 * rh + r) * 16 + i] = sp[r];
        }
    }
}

// ======================================================================= intra-chunk kernel
// GATE: the gate form (kda_gate_kind); NORM: unit-length keys and/or queries (per a.flags).
// tmap_g is the gate tile map: log_alpha [64][128] fp32 (CHANNEL) or f [64][128] bf16
// (FUSED); the scalar gate is read like beta, and no gate is read without decay.
template <int GATE, bool NORM>
__global__ void __launch_bounds__(NTHR, 2)
    kda_chunk_intra_kernel(KdaChunkArgs a, uint8_t *ws, const int32_t *slot_base,
                           const __grid_constant__ CUtensorMap tmap_g, const __grid_constant__ CUtensorMap tmap_k,
                           const __grid_constant__ CUtensorMap tmap_q) {
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u);   // stays a shared-space pointer
    __shared__ uint64_t bar_ap, bar_p, bar_w, bar_in;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

    // The scan may be scheduled once every CTA of this grid has started (it waits for this
    // grid's completion before it reads the workspace).
    asm volatile("griddepcontrol.launch_dependents;");
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H, h = blockIdx.y;
    const int slot = blockIdx.x;
    int n, ci;
    if (slot_base == nullptr) {
        const int per = (a.T + CH - 1) / CH;
        n = slot / per;
        ci = slot - n * per;
        if (n >= a.N) return;
    } else {
        if (slot >= slot_base[a.N]) return;
        int lo = 0, hi = a.N - 1;               // last n with slot_base[n] <= slot
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (slot_base[mid] <= slot) lo = mid; else hi = mid - 1;
        }
        n = lo;
        ci = slot - slot_base[n];
    }
    int64_t t0, t1;
    kda::seq_bounds(a.cu_seqlens, n, a.T, a.T_total, t0, t1);
    const int64_t c0 = t0 + (int64_t)ci * CH;
    const int nr = (int)(t1 - c0 < CH ? t1 - c0 : CH);
    uint8_t *gslot = ws + ((size_t)slot * H + h) * SLOT_BYTES;

    uint8_t *sKQ = sm + I_KQ, *sKC = sm + I_KC, *sIP = sm + I_KC, *sTP = sm + I_TP;
    float *Am = (float *)(sm + I_AM), *Tm = (float *)(sm + I_TM);
    float *sSC = (float *)(sm + I_SC), *sCP = (float *)(sm + I_CP), *sCA = (float *)(sm + I_CA);
    float *sBeta = (float *)(sm + I_BETA), *sGC = (float *)(sm + I_GC);
    float *sBS = (float *)(sm + I_BS), *sBT = (float *)(sm + I_BT), *sXT = (float *)(sm + I_XT);
    float *sRk = (float *)(sm + I_RK), *sRq = (float *)(sm + I_RQ), *sLa = (float *)(sm + I_LA);
    const float scale = a.scale;

    // The chunk's inputs by TMA, issued by one thread: the gate tile (log_alpha [64][128] fp32,
    // or f [64][128] bf16) into the space of [k gamma; s q gamma] and k [64][128] bf16 into the
    // space of the update operand (both row-major; pass 1 moves them to registers before pass 2
    // overwrites them), q as two 64-column halves in the rm_sw layout into the space of
    // [T'; P T'].  Rows past the chunk's end hold the next tokens (zeros past the last token)
    // and are masked where they are read.
    uint8_t *sQ = sTP;
    if (tid == 0) {
        mbar_init(&bar_ap, 1);
        mbar_init(&bar_p, 1);
        mbar_init(&bar_w, 1);
        mbar_init(&bar_in, 1);
        mbar_init_fence();
        s_abort = 0;
        constexpr uint32_t gate_bytes = GATE == kda::GATE_CHANNEL ? 32768u : (GATE == kda::GATE_FUSED ? 16384u : 0u);
        mbar_arrive_expect_tx(&bar_in, 32768u + gate_bytes);
        if (gate_bytes) tma_load_3d(sKQ, &tmap_g, 0, h, (int)c0, &bar_in);
        tma_load_3d(sKC, &tmap_k, 0, h, (int)c0, &bar_in);
        tma_load_3d(sQ, &tmap_q, 0, h, (int)c0, &bar_in);
        tma_load_3d(sQ + 8192, &tmap_q, 64, h, (int)c0, &bar_in);
    }
    if (tid < CH) {
        sBeta[tid] = tid < nr ? kda::beta_of(a.beta[(size_t)(c0 + tid) * H + h], a.flags) : 0.f;
        if (GATE == kda::GATE_SCALAR)
            sLa[tid] = tid < nr ? static_cast<const float *>(a.gate)[(size_t)(c0 + tid) * H + h] : 0.f;
    }
    if (warp == 0) tmem_alloc(&s_tmem, 256);
    __syncthreads();                     // the barriers are initialised before anyone waits
    if (!mbar_wait(&bar_in, 0, kWaitCycles)) s_abort = 1;

    // Unit-length keys / queries: 1 / ||x_r|| per row, four threads per row (k row-major in the
    // update operand's space, q in the rm_sw layout); read in pass 2 after pass 1's barrier.
    if (NORM) {
        const int r = tid >> 2, qd = tid & 3;
        float kk = 0.f, qq = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const uint4 kw = *(const uint4 *)(sKC + r * 256 + qd * 64 + m * 16);
            const uint4 qw = *(const uint4 *)(sQ + (qd >> 1) * 8192 + r * 128 + ((((qd & 1) * 4 + m) ^ (r & 7)) << 4));
            const uint32_t kk4[4] = {kw.x, kw.y, kw.z, kw.w}, qq4[4] = {qw.x, qw.y, qw.z, qw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 x = unpack_bf16(kk4[e]), y = unpack_bf16(qq4[e]);
                kk = fmaf(x.x, x.x, fmaf(x.y, x.y, kk));
                qq = fmaf(y.x, y.x, fmaf(y.y, y.y, qq));
            }
        }
        kk += __shfl_xor_sync(0xffffffffu, kk, 1);
        kk += __shfl_xor_sync(0xffffffffu, kk, 2);
        qq += __shfl_xor_sync(0xffffffffu, qq, 1);
        qq += __shfl_xor_sync(0xffffffffu, qq, 2);
        if (qd == 0) {
            sRk[r] = (a.flags & kda::FLAG_NORM_K) ? 1.f / fmaxf(sqrtf(kk), 1e-12f) : 1.f;
            sRq[r] = (a.flags & kda::FLAG_NORM_Q) ? 1.f / fmaxf(sqrtf(qq), 1e-12f) : 1.f;
        }
    }

    // E2 thread mapping: channels {c2, c2 + 1} of 16-row block eb.
    const int c2 = 2 * (tid & 63), eb = tid >> 6;
    float2 la[16];
    uint32_t kr2[16];
    float2 eA = make_float2(0.f, 0.f), dtb = make_float2(0.f, 0.f);   // e^A_log, dt_bias of the two channels
    if (GATE == kda::GATE_FUSED) {
        const float2 alog = *reinterpret_cast<const float2 *>(a.A_log + (size_t)h * DK + c2);
        eA = make_float2(expf(alog.x), expf(alog.y));
        dtb = *reinterpret_cast<const float2 *>(a.dt_bias + (size_t)h * DK + c2);
    }
#pragma unroll
    for (int rr = 0; rr < 16; ++rr) {
        const int r = 16 * eb + rr;
        const bool ok = r < nr;
        if (GATE == kda::GATE_CHANNEL) {
            la[rr] = ok ? *reinterpret_cast<const float2 *>(sKQ + 4 * (r * DK + c2)) : make_float2(0.f, 0.f);
        } else if (GATE == kda::GATE_FUSED) {
            const float2 f = unpack_bf16(*reinterpret_cast<const uint32_t *>(sKQ + 2 * (r * DK + c2)));
            la[rr] = ok ? make_float2(kda::fused_log_alpha_e(f.x, eA.x, dtb.x), kda::fused_log_alpha_e(f.y, eA.y, dtb.y))
                        : make_float2(0.f, 0.f);
        } else if (GATE == kda::GATE_SCALAR) {
            la[rr] = make_float2(sLa[r], sLa[r]);
        } else {
            la[rr] = make_float2(0.f, 0.f);
        }
        kr2[rr] = ok ? *reinterpret_cast<const uint32_t *>(sKC + 2 * (r * DK + c2)) : 0u;
    }

    // ---------------- E2 pass 1: alpha, per-block sums and products; clear the exact-path sums
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
        const int idx = tid + NTHR * k4;
        sCA[idx] = 0.f;
        sCP[idx] = 0.f;
    }
    {
        float s0 = 0.f, s1 = 0.f, p0 = 1.f, p1 = 1.f;
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            s0 += la[rr].x;
            s1 += la[rr].y;
            la[rr].x = __expf(la[rr].x);
            la[rr].y = __expf(la[rr].y);
            p0 *= la[rr].x;
            p1 *= la[rr].y;
        }
        *reinterpret_cast<float2 *>(&sBS[eb * 128 + c2]) = make_float2(s0, s1);
        *reinterpret_cast<float2 *>(&sBT[eb * 128 + c2]) = make_float2(p0, p1);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem, T_AP = tmem, T_W = tmem + 64;
    const int quarter = warp & 3, half = warp >> 2;
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    const int trow = 32 * quarter + lane;

    float2 gsum = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 bs = *reinterpret_cast<const float2 *>(&sBS[j * 128 + c2]);
        gsum.x += bs.x;
        gsum.y += bs.y;
    }
    const bool fast = __syncthreads_and(gsum.x >= -kChunkSpreadLimit && gsum.y >= -kChunkSpreadLimit);

    // ---------------- E2 pass 2: operands
    {
        float2 gpre = make_float2(1.f, 1.f), ksuf = make_float2(1.f, 1.f);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 bt = *reinterpret_cast<const float2 *>(&sBT[j * 128 + c2]);
            if (j < eb) { gpre.x *= bt.x; gpre.y *= bt.y; }
            if (j > eb) { ksuf.x *= bt.x; ksuf.y *= bt.y; }
        }
        if (fast) {   // k e^-g = k kappa e^{-g_last}
            ksuf.x *= __expf(-gsum.x);
            ksuf.y *= __expf(-gsum.y);
        }
        const uint32_t col_kq = (uint32_t)(c2 >> 6) * 16384u, col_kc = (uint32_t)(c2 >> 6) * 8192u;
        const float2 bs = *reinterpret_cast<const float2 *>(&sBS[eb * 128 + c2]);
        const bool fl0 = bs.x < -kSpreadLimit, fl1 = bs.y < -kSpreadLimit;
        const float rho0 = fast || fl0 ? 1.f : __expf(-0.5f * bs.x);
        const float rho1 = fast || fl1 ? 1.f : __expf(-0.5f * bs.y);
        // the block path's factors, rm_sw tiles: left k in the space of A, right k in the space of
        // k e^-g / [I; P], left s q in place of q (each thread rewrites the elements it read)
        uint8_t *sKL = sm + I_AM, *sKR = sm + I_KC;
        if (fast) {
            // both channels at once on packed fp32 pairs (each lane rounded as the plain product)
            float2 l = make_float2(1.f, 1.f);
            const float2 sc2 = make_float2(scale, scale);
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                const int r = 16 * eb + rr;
                l = __fmul2_rn(l, la[rr]);
                const float2 kv = row_scaled<NORM>(unpack_bf16(kr2[rr]), sRk, r);
                const float2 qv = row_scaled<NORM>(unpack_bf16(r < nr ? *(const uint32_t *)(sQ + rm_sw(r, c2)) : 0u), sRq, r);
                const float2 g = __fmul2_rn(gpre, l);
                const float2 kg = __fmul2_rn(kv, g), qg = __fmul2_rn(__fmul2_rn(sc2, qv), g);
                *(uint32_t *)(sKQ + col_kq + sw128(r, c2 & 63)) = pack_bf16(kg.x, kg.y);
                *(uint32_t *)(sKQ + col_kq + sw128(64 + r, c2 & 63)) = pack_bf16(qg.x, qg.y);
            }
            float2 g = make_float2(1.f, 1.f);
#pragma unroll
            for (int rr = 15; rr >= 0; --rr) {
                const int r = 16 * eb + rr;
                const float2 kv = row_scaled<NORM>(unpack_bf16(kr2[rr]), sRk, r);
                const float2 kk = __fmul2_rn(kv, __fmul2_rn(g, ksuf));
                *(uint32_t *)(sKC + col_kc + sw128(r, c2 & 63)) = pack_bf16(kk.x, kk.y);
                g = __fmul2_rn(g, la[rr]);
            }
        } else {
            // The rescaled factors rho * (prefix product) and rho * (suffix product) are carried
            // as running products that start at rho: they stay in [e^-70, e^70] for a block
            // spread up to kSpreadLimit, where the unscaled products alone would leave fp32's
            // normal range (below e^-87) for spreads past 87 before rho could scale them back.
            float l0 = 1.f, l1 = 1.f, m0 = rho0, m1 = rho1;
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                const int r = 16 * eb + rr;
                l0 *= la[rr].x;
                l1 *= la[rr].y;
                m0 *= la[rr].x;
                m1 *= la[rr].y;
                const float2 kv = row_scaled<NORM>(unpack_bf16(kr2[rr]), sRk, r);
                const float2 qv = row_scaled<NORM>(unpack_bf16(r < nr ? *(const uint32_t *)(sQ + rm_sw(r, c2)) : 0u), sRq, r);
                const float g0 = gpre.x * l0, g1 = gpre.y * l1;
                *(uint32_t *)(sKQ + col_kq + sw128(r, c2 & 63)) = pack_bf16(kv.x * g0, kv.y * g1);
                *(uint32_t *)(sKQ + col_kq + sw128(64 + r, c2 & 63)) = pack_bf16(scale * qv.x * g0, scale * qv.y * g1);
                *(uint32_t *)(sKL + rm_sw(r, c2)) = pack_bf16(kv.x * m0, kv.y * m1);
                *(uint32_t *)(sQ + rm_sw(r, c2)) = pack_bf16(scale * qv.x * m0, scale * qv.y * m1);
            }
            float g0 = 1.f, g1 = 1.f, n0 = rho0, n1 = rho1;
#pragma unroll
            for (int rr = 15; rr >= 0; --rr) {
                const int r = 16 * eb + rr;
                const float2 kv = row_scaled<NORM>(unpack_bf16(kr2[rr]), sRk, r);
                *(uint32_t *)(gslot + SLOT_KC + col_kc + sw128(r, c2 & 63)) =
                    pack_bf16(kv.x * (g0 * ksuf.x), kv.y * (g1 * ksuf.y));
                *(uint32_t *)(sKR + rm_sw(r, c2)) = pack_bf16(kv.x * n0, kv.y * n1);
                g0 *= la[rr].x;
                g1 *= la[rr].y;
                n0 *= la[rr].x;
                n1 *= la[rr].y;
            }
        }
        if (!fast && __syncthreads_or(fl0 || fl1))
            exact_diag_blocks<GATE, NORM>(a, c0, nr, h, sBS, sBeta, sRk, sRq, sCA, sCP);
        if (eb == 0) {
            float2 gc = make_float2(1.f, 1.f);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 bt = *reinterpret_cast<const float2 *>(&sBT[j * 128 + c2]);
                gc.x *= bt.x;
                gc.y *= bt.y;
            }
            *reinterpret_cast<float2 *>(&sGC[c2]) = gc;
            *reinterpret_cast<float2 *>(gslot + SLOT_GC + 4 * c2) = gc;
        }
        if (!fast) {
#pragma unroll
            for (int k5 = 0; k5 < 5; ++k5) {
                const int e = tid + NTHR * k5, p = e >> 7, ch = e & 127, pa = kPairA[p], pb = kPairB[p];
                const float bsa = sBS[pa * 128 + ch], bsb = sBS[pb * 128 + ch];
                const bool fa = bsa < -kSpreadLimit, fb = bsb < -kSpreadLimit;
                float sc;
                if (pa == pb) {
                    sc = fa ? 0.f : 1.f;
                } else {
                    float ex = (fa ? 0.f : 0.5f * bsa) + (fb ? 0.f : 0.5f * bsb);
                    for (int j = pb + 1; j < pa; ++j) ex += sBS[j * 128 + ch];
                    sc = __expf(ex);
                }
                sSC[p * 128 + ch] = sc;
            }
        }
        if (tid == 0) *reinterpret_cast<int *>(gslot + SLOT_FLAG) = fast ? 1 : 0;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---------------- AP: A (fp32, to Am) and P (bf16, lines 64-127 of [I; P])
    if (fast) {
        if (tid == 0) {
            bulk_s2g(gslot + SLOT_KC, sKC, 16384);      // the update operand, already in slot layout
            bulk_commit();
            const uint32_t kq = smem_u32(sKQ), kc = smem_u32(sKC);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(T_AP, desc_sw128(kq + (ks >> 2) * 16384 + 32 * (ks & 3), 16, 1024),
                         desc_sw128(kc + (ks >> 2) * 8192 + 32 * (ks & 3), 16, 1024),
                         idesc_bf16(128, 64, false, false), ks > 0);
            mma_commit(&bar_ap);
        }
        if (!mbar_wait(&bar_ap, 0, kWaitCycles)) s_abort = 1;
        tc_fence_after();
        float v[32];
        tmem_ld32(T_AP + lane_off + half * 32, v);
        tc_fence_before();
        if (tid == 0) bulk_wait_read_all();
        __syncthreads();   // the product and the bulk store have read k e^-g: its space becomes [I; P]
        const int r = trow & 63;
        if (trow < 64) {
            const float bb = sBeta[r];
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const int c = half * 32 + i;
                *reinterpret_cast<float4 *>(Am + r * LF + c) =
                    make_float4(c < r ? bb * v[i] : 0.f, c + 1 < r ? bb * v[i + 1] : 0.f,
                                c + 2 < r ? bb * v[i + 2] : 0.f, c + 3 < r ? bb * v[i + 3] : 0.f);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = half * 32 + i <= r ? v[i] : 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m) *(uint4 *)(sIP + sw128_chunk(trow, 4 * half + m)) = pack8(v + 8 * m);
        }
    } else {
        // 16 x 16 blocks with block-local decay references, warp MMAs on the factors in shared
        // memory.  The results stay in registers until every task has read the factors (A and
        // [I; P] take their space), then go out after a barrier.
        const uint8_t *sKL = sm + I_AM, *sKR = sm + I_KC;
        const int g = lane >> 2, t4 = lane & 3;
        float res[3][2][4];
#pragma unroll
        for (int it = 0; it < 3; ++it) {
            const int task = warp + 8 * it;
            if (task >= 20) break;
            const int mat = task / 10, p = task % 10, pa = kPairA[p], pb = kPairB[p];
            const uint8_t *Ls = mat == 0 ? sKL : sQ;
            float acc[2][2][4] = {};
#pragma unroll 2
            for (int kt = 0; kt < 8; ++kt) {
                const int c = 16 * kt + 2 * t4;
                const uint32_t a0 = *(const uint32_t *)(Ls + rm_sw(16 * pa + g, c));
                const uint32_t a1 = *(const uint32_t *)(Ls + rm_sw(16 * pa + g + 8, c));
                const uint32_t a2 = *(const uint32_t *)(Ls + rm_sw(16 * pa + g, c + 8));
                const uint32_t a3 = *(const uint32_t *)(Ls + rm_sw(16 * pa + g + 8, c + 8));
                const float2 s01 = *reinterpret_cast<const float2 *>(&sSC[p * 128 + c]);
                const float2 s89 = *reinterpret_cast<const float2 *>(&sSC[p * 128 + c + 8]);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int i = 16 * pb + 8 * j + g;
                    const float2 f0 = unpack_bf16(*(const uint32_t *)(sKR + rm_sw(i, c)));
                    const float2 f1 = unpack_bf16(*(const uint32_t *)(sKR + rm_sw(i, c + 8)));
                    mma_m16n8k16(acc[kt & 1][j], a0, a1, a2, a3, pack_bf16(f0.x * s01.x, f0.y * s01.y),
                                 pack_bf16(f1.x * s89.x, f1.y * s89.y));
                }
            }
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) res[it][j][e] = acc[0][j][e] + acc[1][j][e];
        }
        __syncthreads();
#pragma unroll
        for (int it = 0; it < 3; ++it) {
            const int task = warp + 8 * it;
            if (task >= 20) break;
            const int mat = task / 10, p = task % 10, pa = kPairA[p], pb = kPairB[p];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = 16 * pa + g + (e >= 2 ? 8 : 0);
                    const int i = 16 * pb + 8 * j + 2 * t4 + (e & 1);
                    const float val = res[it][j][e];
                    if (mat == 0) {
                        if (pa != pb) Am[r * LF + i] = sBeta[r] * val;
                        else if (i < r) Am[r * LF + i] = sBeta[r] * val + sCA[pa * 256 + (r & 15) * 16 + (i & 15)];
                    } else {
                        float pv = val;
                        if (pa == pb) pv = i <= r ? pv + sCP[pa * 256 + (r & 15) * 16 + (i & 15)] : 0.f;
                        *(__nv_bfloat16 *)(sIP + sw128(64 + r, i)) = __float2bfloat16_rn(pv);
                    }
                }
            }
        }
        //  the six 16 x 16 blocks of P above the diagonal are zero
        for (int o = tid; o < 6 * 256; o += NTHR) {
            const int p = o >> 8;                  // (row block, column block) pairs above the diagonal
            const int pa = p < 3 ? 0 : (p < 5 ? 1 : 2);
            const int pb = p < 3 ? 1 + p : (p < 5 ? p - 1 : 3);
            *(__nv_bfloat16 *)(sIP + sw128(64 + 16 * pa + ((o >> 4) & 15), 16 * pb + (o & 15))) =
                __float2bfloat16_rn(0.f);
        }
    }
    __syncthreads();

    // ---------------- T = (I + A)^{-1}: diagonal 16 x 16 blocks.  Warp w < 4 solves block w by
    //      forward substitution: lane i holds row i of the block of A and column i of T; row r
    //      of A is broadcast from lane r.
    //      Meanwhile warps 4-7 write the identity half of [I; P] and preload the accumulator of
    //      the W product with [0; s q gamma], so that it yields [-W; s q gamma - P W] directly.
    if (warp < 4) {
        const int w = warp, i = lane & 15;
        const float *Ab = Am + (16 * w) * LF + 16 * w;
        float arow[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) arow[m] = Ab[i * LF + m];
        float tcol[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < r; ++m) acc = fmaf(__shfl_sync(0xffffffffu, arow[m], r), tcol[m], acc);
            tcol[r] = r < i ? 0.f : (r == i ? 1.f : -acc);
        }
        if (lane < 16) {
#pragma unroll
            for (int r = 0; r < 16; ++r) Tm[(16 * w + r) * LF + 16 * w + i] = tcol[r];
        }
    } else {
        for (int o = tid - 128; o < 512; o += 128) {       // lines 0-63 of [I; P]: the identity
            const int l = o >> 3, j = o & 7;
            float v8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v8[e] = 8 * j + e == l ? 1.f : 0.f;
            *(uint4 *)(sIP + sw128_chunk(l, j)) = pack8(v8);
        }
#pragma unroll
        for (int part = 0; part < 4; ++part) {             // 32 columns of the W accumulator each
            float v[32];
            if (trow < 64) {
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = 0.f;
            } else {
#pragma unroll
                for (int m = 0; m < 4; ++m) {              // s q gamma of row trow - 64 (KQ tile)
                    const uint4 pk = *(const uint4 *)(sKQ + (part >> 1) * 16384 + sw128_chunk(trow, 4 * (part & 1) + m));
                    const uint32_t w4[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 qq = unpack_bf16(w4[e]);
                        v[8 * m + 2 * e] = qq.x;
                        v[8 * m + 2 * e + 1] = qq.y;
                    }
                }
            }
            tmem_st32(T_W + lane_off + 32 * part, v);
        }
    }
    __syncthreads();
    //      off-diagonal blocks, by distance d = a - b: T_ab = -T_aa sum_{m=b}^{a-1} A_am T_mb,
    //      with tf32 warp MMAs (m16n8k8).  One warp per (block, 8-column half); the partial
    //      product X goes through this warp's slice of the scratch to become a B operand.
    {
        const int g = lane >> 2, t4 = lane & 3;
        for (int d = 1; d < 4; ++d) {
            const int ntask = 2 * (4 - d);
            if (warp < ntask) {
                const int b = warp >> 1, nh = warp & 1, pa = b + d;
                const int col = 16 * b + 8 * nh + g;
                float x[4] = {0.f, 0.f, 0.f, 0.f};
                for (int m = b; m < pa; ++m) {
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        const float *ar = Am + (16 * pa + g) * LF + 16 * m + 8 * kk + t4;
                        const float *tr = Tm + (16 * m + 8 * kk + t4) * LF + col;
                        mma_tf32_m16n8k8(x, to_tf32(ar[0]), to_tf32(ar[8 * LF]), to_tf32(ar[4]),
                                         to_tf32(ar[8 * LF + 4]), to_tf32(tr[0]), to_tf32(tr[4 * LF]));
                    }
                }
                float *xs = sXT + warp * 128;        // X (16 x 8) as [row][8]
                xs[g * 8 + 2 * t4] = x[0];
                xs[g * 8 + 2 * t4 + 1] = x[1];
                xs[(g + 8) * 8 + 2 * t4] = x[2];
                xs[(g + 8) * 8 + 2 * t4 + 1] = x[3];
                __syncwarp();
                float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const float *tr = Tm + (16 * pa + g) * LF + 16 * pa + 8 * kk + t4;
                    mma_tf32_m16n8k8(y, to_tf32(tr[0]), to_tf32(tr[8 * LF]), to_tf32(tr[4]),
                                     to_tf32(tr[8 * LF + 4]), to_tf32(xs[(8 * kk + t4) * 8 + g]),
                                     to_tf32(xs[(8 * kk + t4 + 4) * 8 + g]));
                }
                float *dst = Tm + (16 * pa + g) * LF + 16 * b + 8 * nh + 2 * t4;
                dst[0] = -y[0];
                dst[1] = -y[1];
                dst[8 * LF] = -y[2];
                dst[8 * LF + 1] = -y[3];
            }
            __syncthreads();
        }
    }
    //      T' (lines 0-63 of [T'; P T']), 8 elements at a time
    for (int o = tid; o < 512; o += NTHR) {
        const int l = o >> 3, j = o & 7;
        float v8[8];
        {
            const float4 t0v = *reinterpret_cast<const float4 *>(&Tm[l * LF + 8 * j]);
            const float4 t1v = *reinterpret_cast<const float4 *>(&Tm[l * LF + 8 * j + 4]);
            const float4 b0 = *reinterpret_cast<const float4 *>(&sBeta[8 * j]);
            const float4 b1 = *reinterpret_cast<const float4 *>(&sBeta[8 * j + 4]);
            const float tv[8] = {t0v.x * b0.x, t0v.y * b0.y, t0v.z * b0.z, t0v.w * b0.w,
                                 t1v.x * b1.x, t1v.y * b1.y, t1v.z * b1.z, t1v.w * b1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) v8[e] = 8 * j + e <= l ? tv[e] : 0.f;
            *(uint4 *)(sTP + sw128_chunk(l, j)) = pack8(v8);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---------------- [T'; P T'] = [I; P] T'
    if (tid == 0) {
        const uint32_t ip = smem_u32(sIP), tp = smem_u32(sTP);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_bf16(T_AP, desc_sw128(ip + 32 * ks, 16, 1024), desc_sw128(tp + 2048 * ks, 8192, 1024),
                     idesc_bf16(128, 64, false, true), ks > 0);
        mma_commit(&bar_p);
    }
    if (!mbar_wait(&bar_p, 0, kWaitCycles)) s_abort = 1;
    tc_fence_after();
    if (trow >= 64) {
        float v[32];
        tmem_ld32(T_AP + lane_off + half * 32, v);
#pragma unroll
        for (int m = 0; m < 4; ++m) *(uint4 *)(sTP + sw128_chunk(trow, 4 * half + m)) = pack8(v + 8 * m);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---------------- [-W; s q gamma - P W] = [0; s q gamma] - [T'; P T'] (k gamma); meanwhile
    //      [T'; P T'] goes to the slot
    if (tid == 0) {
        const uint32_t a0 = smem_u32(sTP), b0 = smem_u32(sKQ);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_bf16(T_W, desc_sw128(a0 + 32 * ks, 16, 1024), desc_sw128(b0 + 2048 * ks, 16384, 1024),
                     idesc_bf16(128, 128, false, true, true), 1);
        mma_commit(&bar_w);
    }
    if (tid == 32) {
        bulk_s2g(gslot + SLOT_TP, sTP, 16384);
        bulk_commit();
    }
    if (!mbar_wait(&bar_w, 0, kWaitCycles)) s_abort = 1;
    tc_fence_after();
    //      [-W; s q gamma - P W] -> shared memory in the slot's layout (K-major, 2 x 128 lines;
    //      the space of A and T, no longer needed), then one bulk store to the slot
    uint8_t *sA2 = sm + I_AM;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
        float v[32];
        tmem_ld32(T_W + lane_off + half * 64 + part * 32, v);
#pragma unroll
        for (int m = 0; m < 4; ++m)
            *(uint4 *)(sA2 + half * 16384 + sw128_chunk(trow, 4 * part + m)) = pack8(v + 8 * m);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        bulk_s2g(gslot + SLOT_A2, sA2, 32768);
        bulk_commit();
        bulk_wait_read_all();
    }
    if (tid == 32) bulk_wait_read_all();
    if (s_abort && tid == 0) {
        atomicOr(&g_kda_device_status, 1u);
        mbar_wait(&bar_in, 0, kWaitCycles);   // the input loads must not land in released memory
    }
    __syncthreads();
    if (warp == 0) tmem_free(tmem, 256);
}

// ============================================================================ scan kernel
// One CTA per (sequence, head, 64-column d_v tile); the state tile S (128 x 64 fp32) stays in
// TMEM for the whole sequence.  Warp roles, joined only through mbarriers:
//   warps 0-7  read-out: per chunk c, S out of TMEM (pending decay applied, bf16 copy for the
//              product), then [u; o] out of TMEM: u into shared memory (warps 0, 1, 4, 5 hold
//              TMEM lanes 0-63), o into a staging tile for the store thread (warps 2, 3, 6, 7);
//   warp 8     tensor-core issue (one thread): [u; o] = [T'; P T'] v as soon as the chunk is in
//              shared memory, + [-W; s q gamma - P W] S once S is copied, S += KC^T u once u is;
//   warp 9     loads (one thread): slot c and the v tile of chunk c into stage c & 1 once the
//              state product of chunk c - 2 has released it;
//   warp 10    stores (one thread): o of a full chunk, staged in shared memory by the o warps,
//              to HBM by one TMA store (a partial last chunk is stored directly by the o warps,
//              so no box reaches into the next sequence's tokens).
// [u; o] alternates between two TMEM accumulators so chunk c + 1's first product can start
// while o of chunk c is still being read.
constexpr int SCAN_THREADS = 352;
constexpr int kReadoutThreads = 256;

__global__ void __launch_bounds__(SCAN_THREADS, 1)
    kda_chunk_scan_kernel(KdaChunkArgs a, const uint8_t *ws, const int32_t *slot_base,
                          const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_o) {
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u);   // stays a shared-space pointer
    __shared__ uint64_t bar_ld[2], bar_free[2], bar_ofree[2], bar_sready, bar_uo, bar_uready, bar_s;
    __shared__ uint64_t bar_ostaged[2], bar_obuf[2];
    __shared__ uint32_t s_tmem;
    __shared__ volatile int s_abort;
    __shared__ int s_last, s_issued;      // last commit of the issuing thread (0 none, 1 uo, 2 s); loads issued
    __shared__ uint32_t s_last_par;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H;
    // Varlen: CTAs walk the sequences longest first (the order the slot kernel wrote after the
    // slot offsets); fixed length: in index order.
    const int rank = blockIdx.x / (H * NTILE), rest = blockIdx.x % (H * NTILE);
    const int h = rest / NTILE, tile = rest % NTILE;
    int n = slot_base ? slot_base[a.N + 1 + rank] : rank;
    if (n < 0 || n >= a.N) n = 0;             // not reached: the order is a permutation
    const int pair = n * H + h;
    __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.out);
    int64_t t0, t1;
    kda::seq_bounds(a.cu_seqlens, n, a.T, a.T_total, t0, t1);
    int nchunks = (int)((t1 - t0 + CH - 1) / CH);
    const int base = slot_base ? slot_base[n] : n * ((a.T + CH - 1) / CH);
    if (slot_base && slot_base[n + 1] - base < nchunks) nchunks = slot_base[n + 1] - base;   // malformed offsets
    uint8_t *sS = sm + S_S;

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar_ld[i], 1);
            mbar_init(&bar_free[i], 1);
            mbar_init(&bar_ofree[i], 4);
            mbar_init(&bar_ostaged[i], 4);
            mbar_init(&bar_obuf[i], 1);
        }
        mbar_init(&bar_sready, 8);
        mbar_init(&bar_uo, 1);
        mbar_init(&bar_uready, 4);
        mbar_init(&bar_s, 1);
        mbar_init_fence();
        s_abort = 0;
        s_last = 0;
        s_last_par = 0;
        s_issued = 0;
    }
    if (warp == 0) tmem_alloc(&s_tmem, 256);
    const int quarter = warp & 3, half = (warp >> 2) & 1;
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    const int trow = 32 * quarter + lane;
    const size_t s_base = ((size_t)pair * DK) * DV + (size_t)tile * DVT + half * 32;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem, T_S = tmem;          // [u; o] of chunk c: tmem + 64 + 64 (c & 1)
    // The state row trow is held in TMEM as S / pend: a fast-path chunk's decay is applied
    // when the state is next read.
    float pend = 1.f;
    if (tid < kReadoutThreads) {
        float v[32];
        if (a.S0) {
            const float4 *src = reinterpret_cast<const float4 *>(a.S0 + s_base + (size_t)trow * DV);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 x = src[i];
                v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
        }
        tmem_st32(T_S + lane_off + half * 32, v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // Everything above runs while the intra-chunk grid finishes; the workspace is read below.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 9) {
        // ------------------------------------------------------------------ loads
        if (lane == 0) {
            for (int ci = 0; ci < nchunks; ++ci) {
                const int par = ci & 1;
                if (ci >= 2 && !mbar_wait(&bar_free[par], (uint32_t)((ci - 2) >> 1) & 1u, kWaitCycles)) {
                    s_abort = 1;
                    break;
                }
                if (s_abort) break;
                uint8_t *st = sm + par * S_STAGE;
                const uint8_t *src = ws + ((size_t)(base + ci) * H + h) * SLOT_BYTES;
                mbar_arrive_expect_tx(&bar_ld[par], SLOT_BYTES + 8192);
#pragma unroll
                for (int part = 0; part < 4; ++part)
                    bulk_g2s(st + part * (SLOT_BYTES / 4), src + part * (SLOT_BYTES / 4), SLOT_BYTES / 4,
                             &bar_ld[par]);
                tma_load_3d(st + S_V, &tmap_v, tile * DVT, h, (int)(t0 + (int64_t)ci * CH), &bar_ld[par]);
                s_issued = ci + 1;
            }
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------------ o stores
        if (lane == 0) {
            for (int ci = 0; ci < nchunks; ++ci) {
                const uint32_t b = (uint32_t)(ci & 1);
                if (!mbar_wait(&bar_ostaged[b], (uint32_t)(ci >> 1) & 1u, kWaitCycles) || s_abort) {
                    s_abort = 1;
                    break;
                }
                const int64_t c0 = t0 + (int64_t)ci * CH;
                if (t1 - c0 >= CH) {
                    tma_store_3d(&tmap_o, sm + S_O + b * 8192, tile * DVT, h, (int)c0);
                    bulk_commit();
                }
                bulk_wait_read_all();
                mbar_arrive(&bar_obuf[b]);
            }
            bulk_wait_read_all();
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------------ tensor-core issue
        if (lane == 0) {
            const uint64_t d_tp0 = desc_sw128(smem_u32(sm + SLOT_TP), 16, 1024);
            const uint64_t d_a20 = desc_sw128(smem_u32(sm + SLOT_A2), 16, 1024);
            const uint64_t d_kc0 = desc_sw128(smem_u32(sm + SLOT_KC), 8192, 1024);
            const uint64_t d_v0 = desc_sw128(smem_u32(sm + S_V), 8192, 1024);
            const uint64_t d_s = desc_sw128(smem_u32(sS), 16384, 1024);
            const uint64_t d_stage = (uint64_t)(S_STAGE >> 4);      // one stage further, 16-byte units
            const uint32_t idesc = idesc_bf16(128, DVT, false, true);
            const uint32_t idesc_s = idesc_bf16(128, DVT, true, true);
            // Descriptor start addresses advance in 16-byte units: +2 per 16 columns of a K-major
            // line, +128 per 16 lines of an MN-major tile.
            for (int ci = 0; ci < nchunks; ++ci) {
                const uint32_t par = (uint32_t)(ci & 1);
                const uint32_t T_UO = tmem + 64 + 64 * par;
                const uint64_t so = par ? d_stage : 0;
                bool ok = mbar_wait(&bar_ld[par], (uint32_t)(ci >> 1) & 1u, kWaitCycles);
                if (ok && ci >= 2) ok = mbar_wait(&bar_ofree[par], (uint32_t)((ci - 2) >> 1) & 1u, kWaitCycles);
                if (!ok || s_abort) { s_abort = 1; break; }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(T_UO, d_tp0 + so + 2 * ks, d_v0 + so + 128 * ks, idesc, ks > 0);
                if (!mbar_wait(&bar_sready, par, kWaitCycles) || s_abort) {
                    mma_commit(&bar_uo);          // the products issued above must finish before exit
                    s_last = 1;
                    s_last_par = par;
                    s_abort = 1;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(T_UO, d_a20 + so + (ks >> 2) * 1024 + 2 * (ks & 3), d_s + 128 * ks, idesc, 1);
                mma_commit(&bar_uo);
                s_last = 1;
                s_last_par = par;
                if (!mbar_wait(&bar_uready, par, kWaitCycles) || s_abort) { s_abort = 1; break; }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(T_S, d_kc0 + so + 128 * ks, d_v0 + so + 128 * ks, idesc_s, 1);
                mma_commit(&bar_s);
                mma_commit(&bar_free[par]);
                s_last = 2;
                s_last_par = par;
            }
        }
    } else {
        // ------------------------------------------------------------------ read-out
        const bool u_warp = quarter < 2;
        for (int ci = 0; ci < nchunks; ++ci) {
            const uint32_t par = (uint32_t)(ci & 1);
            uint8_t *st = sm + par * S_STAGE;
            const uint32_t T_UO = tmem + 64 + 64 * par;
            const int64_t c0 = t0 + (int64_t)ci * CH;
            const int nr = (int)(t1 - c0 < CH ? t1 - c0 : CH);
            bool ok = ci == 0 || mbar_wait(&bar_s, (uint32_t)(ci - 1) & 1u, kWaitCycles);
            if (ok) ok = mbar_wait(&bar_ld[par], (uint32_t)(ci >> 1) & 1u, kWaitCycles);
            if (!ok) s_abort = 1;
            if (s_abort) break;
            tc_fence_after();
            // state: apply the pending decay; bf16 copy for the product; store back with this
            // chunk's decay applied now (block path) or deferred (fast path)
            {
                const bool fast = *reinterpret_cast<const int *>(st + SLOT_FLAG) != 0;
                float v[32];
                tmem_ld32(T_S + lane_off + half * 32, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= pend;
#pragma unroll
                for (int m = 0; m < 4; ++m) *(uint4 *)(sS + sw128_chunk(trow, 4 * half + m)) = pack8(v + 8 * m);
                const float gdec = reinterpret_cast<const float *>(st + SLOT_GC)[trow];
                if (!fast) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= gdec;
                }
                tmem_st32(T_S + lane_off + half * 32, v);
                pend = fast ? gdec : 1.f;
            }
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_sready);
            if (!mbar_wait(&bar_uo, par, kWaitCycles)) s_abort = 1;
            if (s_abort) break;
            tc_fence_after();
            float v[32];
            tmem_ld32(T_UO + lane_off + half * 32, v);
            uint4 pk[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) pk[m] = pack8(v + 8 * m);
            if (u_warp) {
                // u -> the v space of this stage (the first product has read v)
#pragma unroll
                for (int m = 0; m < 4; ++m) *(uint4 *)(st + S_V + sw128_chunk(trow, 4 * half + m)) = pk[m];
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_uready);
            } else {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_ofree[par]);
                // o into the staging tile of this chunk parity (free once the TMA store of chunk
                // ci - 2 has read it), or straight to HBM for a partial chunk
                if (nr == CH) {
                    if (ci >= 2 && !mbar_wait(&bar_obuf[par], (uint32_t)((ci - 2) >> 1) & 1u, kWaitCycles))
                        s_abort = 1;
                    uint8_t *so = sm + S_O + par * 8192;
#pragma unroll
                    for (int m = 0; m < 4; ++m) *(uint4 *)(so + sw128_chunk(trow - 64, 4 * half + m)) = pk[m];
                    fence_async_smem();
                } else if (trow - 64 < nr) {
                    uint4 *dst = reinterpret_cast<uint4 *>(
                        og + ((size_t)(c0 + trow - 64) * H + h) * DV + tile * DVT + half * 32);
#pragma unroll
                    for (int m = 0; m < 4; ++m) dst[m] = pk[m];
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_ostaged[par]);
            }
        }
    }
    __syncthreads();

    bool failed = s_abort != 0;
    if (!failed && nchunks > 0) {
        if (s_last != 2 || !mbar_wait(&bar_s, (uint32_t)(nchunks - 1) & 1u, kWaitCycles)) failed = true;
    }
    if (failed) {
        // A wait gave up: record it, give the last committed product and every load still in
        // flight one more bounded wait (shared memory must not be released under them), and
        // leave without writing the state.
        if (tid == 0) atomicOr(&g_kda_device_status, 1u);
        if (s_last == 1) mbar_wait(&bar_uo, s_last_par, kWaitCycles);
        if (s_last == 2) mbar_wait(&bar_s, s_last_par, kWaitCycles);
        for (int ci = s_issued - 2 > 0 ? s_issued - 2 : 0; ci < s_issued; ++ci)
            mbar_wait(&bar_ld[ci & 1], (uint32_t)(ci >> 1) & 1u, kWaitCycles);
    } else if (a.S_final && tid < kReadoutThreads) {
        tc_fence_after();
        float v[32];
        tmem_ld32(T_S + lane_off + half * 32, v);
        float4 *dst = reinterpret_cast<float4 *>(a.S_final + s_base + (size_t)trow * DV);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(pend * v[4 * i], pend * v[4 * i + 1], pend * v[4 * i + 2], pend * v[4 * i + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_free(tmem, 256);
}

// Per-device "already done" flags of the one-time set-up below.  Host threads may call the
// library concurrently: a flag is only a shortcut (the set-up calls are idempotent), so two
// threads that both find it clear both run the set-up, which is harmless.
constexpr int kMaxDevices = 64;
std::atomic<bool> g_configured[kMaxDevices] = {};

using IntraKernel = void (*)(KdaChunkArgs, uint8_t *, const int32_t *, const CUtensorMap, const CUtensorMap,
                             const CUtensorMap);

// The intra-chunk kernel for a gate form and normalisation choice.
IntraKernel intra_kernel_for(int gate_kind, bool norm) {
    switch (gate_kind) {
    case kda::GATE_SCALAR:
        return norm ? kda_chunk_intra_kernel<kda::GATE_SCALAR, true> : kda_chunk_intra_kernel<kda::GATE_SCALAR, false>;
    case kda::GATE_NONE:
        return norm ? kda_chunk_intra_kernel<kda::GATE_NONE, true> : kda_chunk_intra_kernel<kda::GATE_NONE, false>;
    case kda::GATE_FUSED:
        return norm ? kda_chunk_intra_kernel<kda::GATE_FUSED, true> : kda_chunk_intra_kernel<kda::GATE_FUSED, false>;
    default:
        return norm ? kda_chunk_intra_kernel<kda::GATE_CHANNEL, true> : kda_chunk_intra_kernel<kda::GATE_CHANNEL, false>;
    }
}

cudaError_t configure(int dev) {
    if (dev >= 0 && dev < kMaxDevices && g_configured[dev].load(std::memory_order_acquire)) return cudaSuccess;
    cudaError_t e = cudaSuccess;
    for (int g = 0; g < 4; ++g)
        for (int nm = 0; nm < 2; ++nm) {
            e = cudaFuncSetAttribute(intra_kernel_for(g, nm != 0), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kIntraSmem);
            if (e != cudaSuccess) return e;
        }
    e = cudaFuncSetAttribute(kda_chunk_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kScanSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices) g_configured[dev].store(true, std::memory_order_release);
    return cudaSuccess;
}

// Tensor map of v or o viewed as [T_total][H][d_v] bf16: boxes of 64 d_v columns x 1 head x
// 64 tokens, 128-byte swizzle, so one TMA load gives the scan its v tile in the MMA layout and
// one TMA store writes a chunk's o tile.  Tokens past T_total read as zeros; tokens of the next
// sequence that fill a partial last chunk of v only meet zero columns of [T'; P T'], and o of a
// partial chunk is never stored by TMA.
std::atomic<PFN_cuTensorMapEncodeTiled_v12000> g_encode_tiled{nullptr};

cudaError_t encode_map(const KdaChunkArgs &a, const void *base, CUtensorMapDataType dtype, uint32_t esize,
                       uint32_t box_x, CUtensorMapSwizzle swizzle, CUtensorMap *map);

cudaError_t encode_tok_map(const KdaChunkArgs &a, const void *base, CUtensorMap *map) {
    return encode_map(a, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint32_t)DVT, CU_TENSOR_MAP_SWIZZLE_128B, map);
}

// Tensor map of a [T_total][H][128] token tensor with boxes of box_x elements x 1 head x 64 tokens.
cudaError_t encode_map(const KdaChunkArgs &a, const void *base, CUtensorMapDataType dtype, uint32_t esize,
                       uint32_t box_x, CUtensorMapSwizzle swizzle, CUtensorMap *map) {
    memset(map, 0, sizeof(*map));
    if (a.T_total == 0) return cudaSuccess;       // no chunk: the map is never read
    PFN_cuTensorMapEncodeTiled_v12000 encode = g_encode_tiled.load(std::memory_order_acquire);
    if (encode == nullptr) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || fn == nullptr) return cudaErrorNotSupported;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        g_encode_tiled.store(encode, std::memory_order_release);
    }
    static_assert(DK == DV, "one token-tensor layout for q, k, log_alpha, v and o");
    const cuuint64_t dims[3] = {(cuuint64_t)DV, (cuuint64_t)a.H, (cuuint64_t)a.T_total};
    const cuuint64_t strides[2] = {(cuuint64_t)DV * esize, (cuuint64_t)a.H * DV * esize};
    const cuuint32_t box[3] = {box_x, 1, (cuuint32_t)CH};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = encode(map, dtype, 3, const_cast<void *>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int64_t max_slots_of(const KdaChunkArgs &a) {
    return a.cu_seqlens ? (a.T_total + CH - 1) / CH + a.N : (int64_t)a.N * ((a.T + CH - 1) / CH);
}
size_t head_bytes_of(const KdaChunkArgs &a) {      // slot offsets [N + 1], order [N]
    return ((size_t)(2 * a.N + 1) * sizeof(int32_t) + 1023) & ~(size_t)1023;
}

}  // namespace

bool kda_chunk_tc_supports(int dk, int dv) { return dk == DK && dv == DV; }

size_t kda_chunk_tc_workspace_bytes(const KdaChunkArgs &a) {
    return head_bytes_of(a) + (size_t)max_slots_of(a) * a.H * SLOT_BYTES;
}

cudaError_t kda_launch_chunk_tc_ws(const KdaChunkArgs &a, void *ws, cudaStream_t stream) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = configure(dev)) != cudaSuccess) return e;
    const int64_t max_slots = max_slots_of(a);
    int32_t *slot_base = a.cu_seqlens ? static_cast<int32_t *>(ws) : nullptr;
    uint8_t *slots = static_cast<uint8_t *>(ws) + head_bytes_of(a);
    if (max_slots > 0) {
        CUtensorMap tmap_g, tmap_k, tmap_q;
        memset(&tmap_g, 0, sizeof(tmap_g));          // never read by the scalar and no-decay forms
        if (a.gate_kind == kda::GATE_CHANNEL &&
            (e = encode_map(a, a.gate, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, DK, CU_TENSOR_MAP_SWIZZLE_NONE,
                            &tmap_g)) != cudaSuccess)
            return e;
        if (a.gate_kind == kda::GATE_FUSED &&
            (e = encode_map(a, a.gate, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, CU_TENSOR_MAP_SWIZZLE_NONE,
                            &tmap_g)) != cudaSuccess)
            return e;
        if ((e = encode_map(a, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, CU_TENSOR_MAP_SWIZZLE_NONE,
                            &tmap_k)) != cudaSuccess)
            return e;
        if ((e = encode_tok_map(a, a.q, &tmap_q)) != cudaSuccess) return e;
        if (a.cu_seqlens)
            kda_chunk_slots_kernel<<<1, kSortMax, 0, stream>>>(a.cu_seqlens, a.N, a.T_total, max_slots,
                                                                slot_base, slot_base + a.N + 1);
        const dim3 grid((unsigned)max_slots, (unsigned)a.H);
        const bool norm = (a.flags & (kda::FLAG_NORM_K | kda::FLAG_NORM_Q)) != 0;
        intra_kernel_for(a.gate_kind, norm)<<<grid, NTHR, kIntraSmem, stream>>>(a, slots, slot_base, tmap_g,
                                                                                 tmap_k, tmap_q);
    }
    CUtensorMap tmap_v, tmap_o;
    if ((e = encode_tok_map(a, a.v, &tmap_v)) != cudaSuccess) return e;
    if ((e = encode_tok_map(a, a.out, &tmap_o)) != cudaSuccess) return e;
    // Launched with programmatic stream serialisation: its CTAs may start (barrier set-up, TMEM
    // allocation, S0 into TMEM) while the last intra-chunk CTAs run; the kernel waits for
    // that grid before it reads the workspace.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((int64_t)a.N * a.H * NTILE));
    cfg.blockDim = dim3(SCAN_THREADS);
    cfg.dynamicSmemBytes = kScanSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = max_slots > 0 ? 1 : 0;   // without the intra grid, an ordinary launch
    if ((e = cudaLaunchKernelEx(&cfg, kda_chunk_scan_kernel, a, static_cast<const uint8_t *>(slots),
                                static_cast<const int32_t *>(slot_base), tmap_v, tmap_o)) != cudaSuccess)
        return e;
    return cudaGetLastError();
}

cudaError_t kda_launch_chunk_tc(const KdaChunkArgs &a, cudaStream_t stream) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = configure(dev)) != cudaSuccess) return e;
    if ((e = kda_keep_pool_memory(dev)) != cudaSuccess) return e;
    void *ws = nullptr;
    if ((e = cudaMallocAsync(&ws, kda_chunk_tc_workspace_bytes(a), stream)) != cudaSuccess) return e;
    e = kda_launch_chunk_tc_ws(a, ws, stream);
    const cudaError_t f = cudaFreeAsync(ws, stream);
    return e != cudaSuccess ? e : f;
}

// Self-test of the bounded device waits: one thread waits on an mbarrier that nothing arrives
// at, gives up after `limit_cycles` SM clock cycles and records the timeout the way the prefill
// kernels do, so that kda_device_status() reports it and the context stays usable.
__global__ void kda_wait_selftest_kernel(long long limit_cycles) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    mbar_init_fence();
    if (!mbar_wait(&bar, 0, limit_cycles)) atomicOr(&g_kda_device_status, 1u);
}

cudaError_t kda_launch_wait_selftest(int limit_us, cudaStream_t stream) {
    int dev = 0, khz = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev)) != cudaSuccess) return e;
    const long long cycles = (long long)limit_us * (khz > 0 ? khz : 2000000) / 1000;
    kda_wait_selftest_kernel<<<1, 32, 0, stream>>>(cycles);
    return cudaGetLastError();
}

cudaError_t kda_read_device_status(unsigned int *status, bool clear) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(status, g_kda_device_status, sizeof(unsigned int));
    if (e != cudaSuccess || !clear || *status == 0) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_kda_device_status, &zero, sizeof(unsigned int));
}
