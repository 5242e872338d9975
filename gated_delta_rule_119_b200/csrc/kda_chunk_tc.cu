// Chunked KDA prefill on the sm_100a tensor cores (bf16 q/k/v, dk = dv = 128, C = 64).
//
// One CTA owns one (sequence, head, 64-column slice of d_v) and walks the
// sequence chunk by chunk, carrying the fp32 state slice S (128 x 64) in
// tensor memory.  Chunk algebra ("22,580" §6.3 WY/UT form with the per-channel
// cumulative decay of its §08/§9.1; all decay factors are products of alphas
// over the steps strictly after the write up to the read):
//
//   A[r][i]  = beta_r sum_c k_rc k_ic D_ric  (i < r),   P[r][i] = s sum_c q_rc k_ic D_ric  (i <= r)
//   T'       = (I + A)^{-1} Diag(beta)
//   W        = T' (k gamma),  u = T' v - W S,  o = (s q gamma) S + P u
//   S       <- Diag(gamma_last) S + (k kappa)^T u
//
// The output is computed from S without waiting for u:
//   o = (s q gamma - P W) S + (P T') v,
// so one tensor-core accumulation produces both u (rows 0-63) and o (rows
// 64-127):  [u; o] = [T'; P T'] v + [-W; s q gamma - P W] S.
//
// Per chunk:
//  E1  q, k (row-major) and the v slice (swizzled) arrive in shared memory by
//      cp.async issued one chunk ahead; log_alpha is prefetched into registers.
//  E2  one thread per (channel, pair of 16-row blocks): alpha = exp(log_alpha),
//      block-local running products, and from them the operands k gamma,
//      k kappa (tensor-core layout) and the factored operands of the 16 x 16
//      blocks of A and P.  A block (a, b) of A is (k f)_a (k h)_b^T times a
//      per-channel scale, where f, h are block-local products rescaled by
//      rho = exp(-sum_block log_alpha / 2) so that every factor stays in
//      [e^-70, e^70].  A diagonal block whose decay spread exceeds that range
//      is handled per channel by exact running products instead.
//  AP  A and P from those factors with warp-level bf16 MMAs (fp32 accumulation).
//  T   T = (I + A)^{-1} by blocked forward substitution in fp32.
//  TC  tcgen05: [T'; P T'] = [I; P] T';  [W; P W] = [T'; P T'] (k gamma); state readout (bf16 copy,
//      decay in place); [u; o] as above; S += (k kappa)^T u.
#include <stdio.h>

#include "kda_common.cuh"
#include "kda_tc_util.cuh"

__device__ unsigned int g_kda_device_status = 0;

namespace {
using namespace kda_tc;

constexpr int CH = 64, DK = 128, DV = 128;
constexpr int DVT = 64;                 // d_v columns per CTA
constexpr int NTILE = DV / DVT;         // CTAs per (sequence, head)
constexpr int NTHR = 256;
constexpr int LP = 136;                 // row pitch (bf16) of the warp-MMA operand tiles
constexpr int LF = 68;                  // row pitch (fp32) of the 64 x 64 matrices
constexpr float kSpreadLimit = 140.f;   // -sum log_alpha over 16 rows beyond which a block is exact-path
constexpr long long kWaitCycles = 4000000000LL;   // about 2 s at B200 clocks
constexpr uint32_t kTmemCols = 256;

// Shared-memory map (bytes from a 1024-byte aligned base).
constexpr uint32_t OFF_V = 0;                       // v slice, then u: 64 lines (MN-major B)
constexpr uint32_t OFF_TP = OFF_V + 8192;           // [T'; P T']: 128 lines (K-major A)
constexpr uint32_t OFF_KQ = OFF_TP + 16384;         // [k gamma; s q gamma]: 2 x 128 lines (K-major A;
                                                    //   lines 0-63 are also the MN-major B of W)
constexpr uint32_t OFF_KC = OFF_KQ + 32768;         // k kappa (block path) or k e^-g (fast path):
                                                    //   2 x 64 lines (MN-major A of the update,
                                                    //   K-major B of A and P on the fast path)
constexpr uint32_t OFF_X = OFF_KC + 16384;          // region X, reused within a chunk:
//   block path, A/P phase: KL @0, KR @17408, QL @34816 (each [64][LP] bf16), SC @52224 ([10][128] fp32)
//   T solve: Tm @16384 ([64][LF] fp32);  then [I; P] @0 (128 lines), S copy @32768 (128 lines),
//   then [-W; Q'] @0 (2 x 128 lines)
constexpr uint32_t X_KL = 0, X_KR = 17408, X_QL = 34816, X_SC = 52224, X_TM = 16384;
constexpr uint32_t X_IP = 0, X_S = 32768, X_A2 = 0, X_SIZE = 57344;
constexpr uint32_t OFF_Q = OFF_X + X_SIZE;          // raw q [64][128] bf16
constexpr uint32_t OFF_K = OFF_Q + 16384;           // raw k
constexpr uint32_t OFF_AM = OFF_K + 16384;          // A [64][LF] fp32
constexpr uint32_t OFF_PM = OFF_AM + 17408;         // P [64][LF] fp32
constexpr uint32_t OFF_SMALL = OFF_PM + 17408;
constexpr uint32_t SM_BETA = OFF_SMALL;             // [64]
constexpr uint32_t SM_GC = SM_BETA + 256;           // [128]   gamma_last
constexpr uint32_t SM_BS = SM_GC + 512;             // [4][128] sum of log_alpha per block
constexpr uint32_t SM_BT = SM_BS + 2048;            // [4][128] product of alpha per block
constexpr uint32_t SM_XT = SM_BT + 2048;            // [6][128] forward-substitution scratch
constexpr uint32_t SM_END = SM_XT + 3072;
constexpr size_t kSmemBytes = SM_END + 1024;        // + alignment slack
static_assert(OFF_X % 1024 == 0 && (OFF_X + X_S) % 1024 == 0 && OFF_KC % 1024 == 0, "tile alignment");
static_assert(X_TM + 17408 <= X_S + 16384 && X_TM >= X_IP + 16384, "T must not meet [I; P]");
static_assert(X_SC + 5120 <= X_SIZE, "scale table inside X");
static_assert(kSmemBytes <= 232448, "shared memory budget");
// Largest decay spread -sum log_alpha over a chunk for the fast path: the factors e^g and e^-g
// then stay within [e^-80, e^80], inside the bf16 / fp32 normal range.
constexpr float kChunkSpreadLimit = 80.f;

__constant__ int kPairA[10] = {0, 1, 1, 2, 2, 2, 3, 3, 3, 3};
__constant__ int kPairB[10] = {0, 0, 1, 0, 1, 2, 0, 1, 2, 3};

__device__ __forceinline__ float bf(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ float2 bf2(const __nv_bfloat16 *p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
}
__device__ __forceinline__ void st_bf2(void *p, float x, float y) {
    *reinterpret_cast<uint32_t *>(p) = pack_bf16(x, y);
}

struct ChunkPos {
    int64_t c0;
    int nr;
};

__device__ __forceinline__ ChunkPos chunk_pos(int64_t t0, int64_t t1, int ci) {
    const int64_t c0 = t0 + (int64_t)ci * CH;
    return {c0, (int)(t1 - c0 < CH ? t1 - c0 : CH)};
}

// Stage q and k rows [c0, c0 + 64) (rows past the sequence end read as zero).
__device__ __forceinline__ void issue_qk(uint8_t *sm, const __nv_bfloat16 *qg, const __nv_bfloat16 *kg,
                                         ChunkPos cp, int H, int h, int tid) {
    for (int idx = tid; idx < 2048; idx += NTHR) {
        const int which = idx >> 10, rem = idx & 1023, r = rem >> 4, j = rem & 15;
        const int rs = r < cp.nr ? r : cp.nr - 1;
        const __nv_bfloat16 *src = (which ? kg : qg) + ((size_t)(cp.c0 + rs) * H + h) * DK + j * 8;
        cp_async16(sm + (which ? OFF_K : OFF_Q) + r * 256 + j * 16, src, r < cp.nr ? 16u : 0u);
    }
}
__device__ __forceinline__ void issue_v(uint8_t *dst, const __nv_bfloat16 *vg, ChunkPos cp, int H,
                                        int h, int tile, int tid) {
    for (int idx = tid; idx < 512; idx += NTHR) {
        const int r = idx >> 3, j = idx & 7;
        const int rs = r < cp.nr ? r : cp.nr - 1;
        const __nv_bfloat16 *src = vg + ((size_t)(cp.c0 + rs) * H + h) * DV + tile * DVT + j * 8;
        cp_async16(dst + sw128_chunk(r, j), src, r < cp.nr ? 16u : 0u);
    }
}
// log_alpha of 16 rows x 2 channels for E2 (zero past the sequence end).
__device__ __forceinline__ void load_la(float2 *la, const float *lag, ChunkPos cp, int H, int h, int b,
                                        int c2) {
#pragma unroll
    for (int rr = 0; rr < 16; ++rr) {
        const int r = 16 * b + rr;
        la[rr] = r < cp.nr ? *reinterpret_cast<const float2 *>(lag + ((size_t)(cp.c0 + r) * H + h) * DK + c2)
                           : make_float2(0.f, 0.f);
    }
}
__device__ __forceinline__ uint4 pack8(const float *v) {
    uint4 pk;
    pk.x = pack_bf16(v[0], v[1]);
    pk.y = pack_bf16(v[2], v[3]);
    pk.z = pack_bf16(v[4], v[5]);
    pk.w = pack_bf16(v[6], v[7]);
    return pk;
}

__global__ void __launch_bounds__(NTHR, 1) kda_chunk_tc_kernel(KdaChunkArgs a) {
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t bar_ap, bar_p, bar_w, bar_uo, bar_s;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

    uint8_t *sV = sm + OFF_V, *sTP = sm + OFF_TP, *sKQ = sm + OFF_KQ, *sKC = sm + OFF_KC;
    uint8_t *sX = sm + OFF_X;
    __nv_bfloat16 *KL = (__nv_bfloat16 *)(sX + X_KL), *KR = (__nv_bfloat16 *)(sX + X_KR);
    __nv_bfloat16 *QL = (__nv_bfloat16 *)(sX + X_QL);
    float *sSC = (float *)(sX + X_SC), *Tm = (float *)(sX + X_TM);
    uint8_t *sIP = sX + X_IP, *sA2 = sX + X_A2, *sS = sX + X_S;
    const __nv_bfloat16 *sQ = (const __nv_bfloat16 *)(sm + OFF_Q);
    const __nv_bfloat16 *sK = (const __nv_bfloat16 *)(sm + OFF_K);
    float *Am = (float *)(sm + OFF_AM), *Pm = (float *)(sm + OFF_PM);
    float *sBeta = (float *)(sm + SM_BETA), *sGC = (float *)(sm + SM_GC);
    float *sBS = (float *)(sm + SM_BS), *sBT = (float *)(sm + SM_BT), *sXT = (float *)(sm + SM_XT);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H;
    const int pair = blockIdx.x / NTILE, tile = blockIdx.x % NTILE;
    const int n = pair / H, h = pair % H;
    const float scale = a.scale;
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(a.q);
    const __nv_bfloat16 *kg = static_cast<const __nv_bfloat16 *>(a.k);
    const __nv_bfloat16 *vg = static_cast<const __nv_bfloat16 *>(a.v);
    __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.out);
    int64_t t0, t1;
    kda::seq_bounds(a.cu_seqlens, n, a.T, a.T_total, t0, t1);
    const int nchunks = (int)((t1 - t0 + CH - 1) / CH);

    // E2 thread mapping: channels {c2, c2 + 1} of 16-row block eb.
    const int c2 = 2 * (tid & 63), eb = tid >> 6;
    float2 la[16];
    float beta_next = 0.f;                      // beta of row tid (< 64) of the chunk to come
    if (nchunks > 0) {
        const ChunkPos cp0 = chunk_pos(t0, t1, 0);
        issue_qk(sm, qg, kg, cp0, H, h, tid);
        load_la(la, a.log_alpha, cp0, H, h, eb, c2);
        if (tid < CH && tid < cp0.nr) beta_next = a.beta[(size_t)(cp0.c0 + tid) * H + h];
    }
    asm volatile("cp.async.commit_group;" ::: "memory");

    if (tid == 0) {
        mbar_init(&bar_ap, 1);
        mbar_init(&bar_p, 1);
        mbar_init(&bar_w, 1);
        mbar_init(&bar_uo, 1);
        mbar_init(&bar_s, 1);
        mbar_init_fence();
        s_abort = 0;
    }
    if (warp == 0) tmem_alloc(&s_tmem, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const uint32_t T_S = tmem, T_UO = tmem + DVT, T_W = tmem + 2 * DVT;
    const int quarter = warp & 3, half = warp >> 2;
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    const int trow = 32 * quarter + lane;       // the TMEM lane (matrix row) this thread serves
    const size_t s_base = ((size_t)pair * DK) * DV + (size_t)tile * DVT + half * 32;
    // The state row trow is stored in TMEM times 1 / pend: the decay of a fast-path chunk is
    // applied when the state is next read.
    float pend = 1.f;

    {   // initial state slice -> TMEM
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

    uint64_t *pending = nullptr;
    uint32_t pending_par = 0;
    for (int ci = 0; ci < nchunks; ++ci) {
        const uint32_t par = (uint32_t)(ci & 1);
        const ChunkPos cp = chunk_pos(t0, t1, ci);
        const int64_t c0 = cp.c0;
        const int nr = cp.nr;

        // ---------------- E1: this chunk's v (needed late); wait for its q, k
        issue_v(sV, vg, cp, H, h, tile, tid);
        asm volatile("cp.async.commit_group;" ::: "memory");
        if (tid < CH) sBeta[tid] = beta_next;
        asm volatile("cp.async.wait_group 1;" ::: "memory");
        __syncthreads();

        // ---------------- E2 pass 1: alpha, per-block sums and products; clear diag(A), diag(P)
#pragma unroll
        for (int k8 = 0; k8 < 8; ++k8) {
            const int idx = tid + NTHR * k8, m = idx >> 10, rem = idx & 1023, blk = rem >> 8;
            (m ? Pm : Am)[(16 * blk + ((rem >> 4) & 15)) * LF + 16 * blk + (rem & 15)] = 0.f;
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
        __syncthreads();
        // Fast path iff every channel's decay spread over the chunk is within the limit.
        float2 gsum = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 bs = *reinterpret_cast<const float2 *>(&sBS[j * 128 + c2]);
            gsum.x += bs.x;
            gsum.y += bs.y;
        }
        const bool fast = __syncthreads_and(gsum.x >= -kChunkSpreadLimit && gsum.y >= -kChunkSpreadLimit);

        // ---------------- E2 pass 2: operands (alpha now in la)
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
            float l0 = 1.f, l1 = 1.f;
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                const int r = 16 * eb + rr;
                l0 *= la[rr].x;
                l1 *= la[rr].y;
                const float2 kv = bf2(&sK[r * 128 + c2]), qv = bf2(&sQ[r * 128 + c2]);
                const float g0 = gpre.x * l0, g1 = gpre.y * l1;
                st_bf2(sKQ + col_kq + sw128(r, c2 & 63), kv.x * g0, kv.y * g1);
                st_bf2(sKQ + col_kq + sw128(64 + r, c2 & 63), scale * qv.x * g0, scale * qv.y * g1);
                if (!fast) {
                    st_bf2(&KL[r * LP + c2], kv.x * (rho0 * l0), kv.y * (rho1 * l1));
                    st_bf2(&QL[r * LP + c2], scale * qv.x * (rho0 * l0), scale * qv.y * (rho1 * l1));
                }
            }
            float g0 = 1.f, g1 = 1.f;
#pragma unroll
            for (int rr = 15; rr >= 0; --rr) {
                const int r = 16 * eb + rr;
                const float2 kv = bf2(&sK[r * 128 + c2]);
                st_bf2(sKC + col_kc + sw128(r, c2 & 63), kv.x * (g0 * ksuf.x), kv.y * (g1 * ksuf.y));
                if (!fast) st_bf2(&KR[r * LP + c2], kv.x * (rho0 * g0), kv.y * (rho1 * g1));
                g0 *= la[rr].x;
                g1 *= la[rr].y;
            }
            if (!fast && (fl0 || fl1)) {
                // Exact diagonal-block contribution of a flagged channel (running products).
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    if (!(cc ? fl1 : fl0)) continue;
                    const int ch = c2 + cc;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float ki = bf(&sK[(16 * eb + i) * 128 + ch]);
                        float f = 1.f;
#pragma unroll
                        for (int r = i; r < 16; ++r) {
                            if (r > i) f *= cc ? la[r].y : la[r].x;
                            const int R = 16 * eb + r, I = 16 * eb + i;
                            const float kd = ki * f;
                            if (r > i) atomicAdd(&Am[R * LF + I], sBeta[R] * bf(&sK[R * 128 + ch]) * kd);
                            atomicAdd(&Pm[R * LF + I], scale * bf(&sQ[R * 128 + ch]) * kd);
                        }
                    }
                }
            }
            if (eb == 0) {
                float2 gc = make_float2(1.f, 1.f);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 bt = *reinterpret_cast<const float2 *>(&sBT[j * 128 + c2]);
                    gc.x *= bt.x;
                    gc.y *= bt.y;
                }
                *reinterpret_cast<float2 *>(&sGC[c2]) = gc;
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
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---------------- AP: A and P
        if (fast) {
            //  [A_raw; P_raw] = [k gamma; s q gamma] (k e^-g)^T on the tensor cores
            if (tid == 0) {
                const uint32_t kq = smem_u32(sKQ), kc = smem_u32(sKC);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(T_UO, desc_sw128(kq + (ks >> 2) * 16384 + 32 * (ks & 3), 16, 1024),
                             desc_sw128(kc + (ks >> 2) * 8192 + 32 * (ks & 3), 16, 1024),
                             idesc_bf16(128, 64, false, false), ks > 0);
                mma_commit(&bar_ap);
            }
            if (!mbar_wait(&bar_ap, par, kWaitCycles)) s_abort = 1;
            tc_fence_after();
            float v[32];
            tmem_ld32(T_UO + lane_off + half * 32, v);
            const int r = trow & 63;
            float *dst = (trow < 64 ? Am : Pm) + r * LF + half * 32;
            const float bscale = trow < 64 ? sBeta[r] : 1.f;
            const int lim = trow < 64 ? r : r + 1;     // A strictly lower, P lower with diagonal
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const int c = half * 32 + i;
                *reinterpret_cast<float4 *>(dst + i) =
                    make_float4(c < lim ? bscale * v[i] : 0.f, c + 1 < lim ? bscale * v[i + 1] : 0.f,
                                c + 2 < lim ? bscale * v[i + 2] : 0.f, c + 3 < lim ? bscale * v[i + 3] : 0.f);
            }
        } else {
            //  16 x 16 blocks with block-local decay references, warp MMAs
            const int g = lane >> 2, t4 = lane & 3;
            for (int task = warp; task < 20; task += 8) {
                const int mat = task / 10, p = task % 10, pa = kPairA[p], pb = kPairB[p];
                const __nv_bfloat16 *Ls = mat == 0 ? KL : QL;
                float acc[2][2][4] = {};
#pragma unroll
                for (int kt = 0; kt < 8; ++kt) {
                    const int c = 16 * kt + 2 * t4;
                    const uint32_t a0 = *(const uint32_t *)&Ls[(16 * pa + g) * LP + c];
                    const uint32_t a1 = *(const uint32_t *)&Ls[(16 * pa + g + 8) * LP + c];
                    const uint32_t a2 = *(const uint32_t *)&Ls[(16 * pa + g) * LP + c + 8];
                    const uint32_t a3 = *(const uint32_t *)&Ls[(16 * pa + g + 8) * LP + c + 8];
                    const float2 s01 = *reinterpret_cast<const float2 *>(&sSC[p * 128 + c]);
                    const float2 s89 = *reinterpret_cast<const float2 *>(&sSC[p * 128 + c + 8]);
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int i = 16 * pb + 8 * j + g;
                        const float2 f0 = unpack_bf16(*(const uint32_t *)&KR[i * LP + c]);
                        const float2 f1 = unpack_bf16(*(const uint32_t *)&KR[i * LP + c + 8]);
                        mma_m16n8k16(acc[kt & 1][j], a0, a1, a2, a3, pack_bf16(f0.x * s01.x, f0.y * s01.y),
                                     pack_bf16(f1.x * s89.x, f1.y * s89.y));
                    }
                }
#pragma unroll
                for (int j = 0; j < 2; ++j) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int r = 16 * pa + g + (e >= 2 ? 8 : 0);
                        const int i = 16 * pb + 8 * j + 2 * t4 + (e & 1);
                        const float val = acc[0][j][e] + acc[1][j][e];
                        if (mat == 0) {
                            if (pa != pb) Am[r * LF + i] = sBeta[r] * val;
                            else if (i < r) Am[r * LF + i] += sBeta[r] * val;
                        } else {
                            if (pa != pb) Pm[r * LF + i] = val;
                            else if (i <= r) Pm[r * LF + i] += val;
                        }
                    }
                }
            }
        }
        __syncthreads();
        if (s_abort) { pending = &bar_ap; pending_par = par; break; }

        // ---------------- T = (I + A)^{-1}: diagonal 16 x 16 blocks.  Warp w < 4 solves block w:
        //      lane i and lane i + 16 both carry column i; each sums half of every row's terms
        //      (even / odd m) and one shuffle joins them.
        if (warp < 4) {
            const int w = warp, i = lane & 15, odd = lane >> 4;
            const float *Ab = Am + (16 * w) * LF + 16 * w;
            float tc[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                for (int m = 0; m < r; ++m) {
                    if ((m & 1) == odd && m >= i) {
                        if (m & 2) acc1 = fmaf(Ab[r * LF + m], tc[m], acc1);
                        else acc0 = fmaf(Ab[r * LF + m], tc[m], acc0);
                    }
                }
                const float part = acc0 + acc1;
                const float tot = part + __shfl_xor_sync(0xffffffffu, part, 16);
                tc[r] = r < i ? 0.f : (r == i ? 1.f : -tot);
            }
            if (!odd) {
#pragma unroll
                for (int r = 0; r < 16; ++r) Tm[(16 * w + r) * LF + 16 * w + i] = tc[r];
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
                    const int col = 16 * b + 8 * nh + g;      // B-operand column of this lane
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
        //      T' (lines 0-63 of [T'; P T']) and [I; P] as tensor-core operands, 8 elements at a time
        for (int o = tid; o < 1536; o += NTHR) {
            const int l = o >> 3, j = o & 7;     // l < 64: T' line; else [I; P] line l - 64
            float v8[8];
            if (l < 64) {
                const float4 t0 = *reinterpret_cast<const float4 *>(&Tm[l * LF + 8 * j]);
                const float4 t1 = *reinterpret_cast<const float4 *>(&Tm[l * LF + 8 * j + 4]);
                const float4 b0 = *reinterpret_cast<const float4 *>(&sBeta[8 * j]);
                const float4 b1 = *reinterpret_cast<const float4 *>(&sBeta[8 * j + 4]);
                const float tv[8] = {t0.x * b0.x, t0.y * b0.y, t0.z * b0.z, t0.w * b0.w,
                                     t1.x * b1.x, t1.y * b1.y, t1.z * b1.z, t1.w * b1.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) v8[e] = 8 * j + e <= l ? tv[e] : 0.f;
                *(uint4 *)(sTP + sw128_chunk(l, j)) = pack8(v8);
            } else {
                const int pl = l - 64;          // line of [I; P]
                if (pl < 64) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) v8[e] = 8 * j + e == pl ? 1.f : 0.f;
                } else {
                    const int r = pl - 64;
                    const float4 p0 = *reinterpret_cast<const float4 *>(&Pm[r * LF + 8 * j]);
                    const float4 p1 = *reinterpret_cast<const float4 *>(&Pm[r * LF + 8 * j + 4]);
                    const float pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) v8[e] = 8 * j + e <= r ? pv[e] : 0.f;
                }
                *(uint4 *)(sIP + sw128_chunk(pl, j)) = pack8(v8);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---------------- TC: [T'; P T'] = [I; P] T'   (into the [u; o] columns, free here)
        if (tid == 0) {
            const uint32_t ip = smem_u32(sIP), tp = smem_u32(sTP);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(T_UO, desc_sw128(ip + 32 * ks, 16, 1024), desc_sw128(tp + 2048 * ks, 8192, 1024),
                         idesc_bf16(128, 64, false, true), ks > 0);
            mma_commit(&bar_p);
        }
        //      state slice: apply the pending decay; bf16 copy for the MMAs; store back with this
        //      chunk's decay applied now (block path) or deferred (fast path).
        {
            float v[32];
            tmem_ld32(T_S + lane_off + half * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= pend;
#pragma unroll
            for (int m = 0; m < 4; ++m) *(uint4 *)(sS + sw128_chunk(trow, 4 * half + m)) = pack8(v + 8 * m);
            const float gdec = sGC[trow];
            if (!fast) {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= gdec;
            }
            tmem_st32(T_S + lane_off + half * 32, v);
            pend = fast ? gdec : 1.f;
        }
        if (!mbar_wait(&bar_p, par, kWaitCycles)) s_abort = 1;
        tc_fence_after();
        if (trow >= 64) {
            float v[32];
            tmem_ld32(T_UO + lane_off + half * 32, v);
#pragma unroll
            for (int m = 0; m < 4; ++m) *(uint4 *)(sTP + sw128_chunk(trow, 4 * half + m)) = pack8(v + 8 * m);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (s_abort) { pending = &bar_p; pending_par = par; break; }
        tc_fence_after();

        // ---------------- TC: [W; P W] = [T'; P T'] (k gamma)
        if (tid == 0) {
            const uint32_t a0 = smem_u32(sTP), b0 = smem_u32(sKQ);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(T_W, desc_sw128(a0 + 32 * ks, 16, 1024), desc_sw128(b0 + 2048 * ks, 16384, 1024),
                         idesc_bf16(128, 128, false, true), ks > 0);
            mma_commit(&bar_w);
        }
        // While the tensor core works: q, k of the next chunk replace this chunk's (dead since
        // E2), and its log_alpha and beta go to registers.
        if (ci + 1 < nchunks) {
            const ChunkPos cn = chunk_pos(t0, t1, ci + 1);
            issue_qk(sm, qg, kg, cn, H, h, tid);
            load_la(la, a.log_alpha, cn, H, h, eb, c2);
            beta_next = (tid < CH && tid < cn.nr) ? a.beta[(size_t)(cn.c0 + tid) * H + h] : 0.f;
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        if (!mbar_wait(&bar_w, par, kWaitCycles)) s_abort = 1;
        tc_fence_after();
        //      [-W; s q gamma - P W] -> tensor-core operand (K-major, 2 x 128 lines)
        {
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                float v[32];
                tmem_ld32(T_W + lane_off + half * 64 + part * 32, v);
                if (trow >= 64) {
#pragma unroll
                    for (int m = 0; m < 4; ++m) {    // s q gamma of row trow - 64, from the KQ tile
                        const uint4 pk = *(const uint4 *)(sKQ + half * 16384 + sw128_chunk(trow, 4 * part + m));
                        const uint32_t w4[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 qq = unpack_bf16(w4[e]);
                            v[8 * m + 2 * e] = qq.x - v[8 * m + 2 * e];
                            v[8 * m + 2 * e + 1] = qq.y - v[8 * m + 2 * e + 1];
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = -v[i];
                }
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    *(uint4 *)(sA2 + half * 16384 + sw128_chunk(trow, 4 * part + m)) = pack8(v + 8 * m);
            }
        }
        asm volatile("cp.async.wait_group 1;" ::: "memory");    // this chunk's v slice
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (s_abort) { pending = &bar_w; pending_par = par; break; }
        tc_fence_after();

        // ---------------- TC: [u; o] = [T'; P T'] v + [-W; Q'] S
        if (tid == 0) {
            const uint32_t idesc = idesc_bf16(128, DVT, false, true);
            const uint32_t tp = smem_u32(sTP), vv = smem_u32(sV), a2 = smem_u32(sA2), ss = smem_u32(sS);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(T_UO, desc_sw128(tp + 32 * ks, 16, 1024), desc_sw128(vv + 2048 * ks, 8192, 1024),
                         idesc, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(T_UO, desc_sw128(a2 + (ks >> 2) * 16384 + 32 * (ks & 3), 16, 1024),
                         desc_sw128(ss + 2048 * ks, 16384, 1024), idesc, 1);
            mma_commit(&bar_uo);
        }
        if (!mbar_wait(&bar_uo, par, kWaitCycles)) s_abort = 1;
        tc_fence_after();
        {
            float v[32];
            tmem_ld32(T_UO + lane_off + half * 32, v);
            uint4 pk[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) pk[m] = pack8(v + 8 * m);
            if (trow < 64) {
#pragma unroll
                for (int m = 0; m < 4; ++m) *(uint4 *)(sV + sw128_chunk(trow, 4 * half + m)) = pk[m];
            } else if (trow - 64 < nr) {
                uint4 *dst = reinterpret_cast<uint4 *>(
                    og + ((size_t)(c0 + trow - 64) * H + h) * DV + tile * DVT + half * 32);
#pragma unroll
                for (int m = 0; m < 4; ++m) dst[m] = pk[m];
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (s_abort) { pending = &bar_uo; pending_par = par; break; }
        tc_fence_after();

        // ---------------- TC: S += (k kappa)^T u  (block path)  or  (k e^-g)^T u  (fast path)
        if (tid == 0) {
            const uint32_t kc = smem_u32(sKC), uu = smem_u32(sV);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(T_S, desc_sw128(kc + 2048 * ks, 8192, 1024), desc_sw128(uu + 2048 * ks, 8192, 1024),
                         idesc_bf16(128, DVT, true, true), 1);
            mma_commit(&bar_s);
        }
        if (!mbar_wait(&bar_s, par, kWaitCycles)) s_abort = 1;
        tc_fence_after();
        __syncthreads();
        if (s_abort) { pending = &bar_s; pending_par = par; break; }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");

    if (pending) {
        // A tensor-core wait gave up: record it, give the in-flight work one more
        // bounded wait, and leave without writing the state.
        if (tid == 0) atomicOr(&g_kda_device_status, 1u);
        mbar_wait(pending, pending_par, kWaitCycles);
    } else if (a.S_final) {
        float v[32];
        tmem_ld32(T_S + lane_off + half * 32, v);
        float4 *dst = reinterpret_cast<float4 *>(a.S_final + s_base + (size_t)trow * DV);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(pend * v[4 * i], pend * v[4 * i + 1], pend * v[4 * i + 2], pend * v[4 * i + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_free(tmem, kTmemCols);
}

}  // namespace

bool kda_chunk_tc_supports(int dk, int dv) { return dk == DK && dv == DV; }

cudaError_t kda_launch_chunk_tc(const KdaChunkArgs &a, cudaStream_t stream) {
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !configured[dev]) {
        e = cudaFuncSetAttribute(kda_chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev] = true;
    }
    const unsigned grid = (unsigned)((int64_t)a.N * a.H * NTILE);
    kda_chunk_tc_kernel<<<grid, NTHR, kSmemBytes, stream>>>(a);
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
