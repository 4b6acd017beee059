// replay.cu -- replay decode: SSM state kept as a checkpoint plus the SSM
// inputs of the tokens since it (sm_100a).
//
// Follows "ReplaySSM: Cache SSM Inputs, Not State" (abstract): unrolling the
// recurrence lets a slot's state be represented by a checkpoint and a short
// buffer of recent SSM inputs. Outputs are computed by replaying the buffer
// from the checkpoint, and the checkpoint is rewritten only once every W
// tokens, so most steps read a checkpoint and write nothing of it. A bf16 copy
// of the checkpoint serves the outputs of the other steps, while the fp32
// checkpoint alone feeds the recurrent update, so the copy's rounding never
// enters later states. The per-token math is that of tp_builder.py
// (TensorRT-Model-Connect, Mamba family), _add_mamba_tp_layer, exactly as in
// the eager decode kernel: the same conv, softplus, exponentials and packed
// fp32x2 update, in the same order, so a checkpoint written here is bit-for-bit
// the state eager decode would hold after the same tokens.
//
// For Mamba-1 the SSM inputs of a (token, channel) are two scalars, delta and
// delta * xc (B is shared by the row and buffered once per token), so a
// buffered token costs 8 bytes per channel against 64 bytes of fp32 state.
// Per (row, channel), a step with j buffered tokens moves
//   32 B (bf16 copy) + 8j B (buffer) + 8 B (new entry) + 20 B (conv state, x, dt, z, y);
// a checkpoint step (j = W-1) moves 64 B in, 64 + 32 B out, 8j B of buffer and
// 20 B. At W = 4 that averages 102 B against eager decode's 148 B, for 2.5
// times the exponentials (j + 1 tokens are replayed).
//
// The buffer length of a slot is shared by all channel blocks of its row. A
// CTA reads it before it issues the row's loads; after finishing the row it
// takes a ticket (one atomic per CTA and row), and the CTA that takes the last
// ticket writes the new length and resets the ticket, so no CTA can observe a
// length written during the same launch. Atomics only count tickets; they
// take no part in the arithmetic.
#include "common.cuh"
#include "tma.cuh"

namespace ssm {

__device__ int g_replay_status = 0;

namespace {

constexpr int kN = 16;
constexpr int kCh = 128;       // channels (threads) per CTA
constexpr int kStages = 3;     // rows in flight per CTA

struct RParams {
    void *conv_state;
    float *ckpt;
    __nv_bfloat16 *ckpt_lo;
    float *buf;
    float *bufB;
    int32_t *len;
    uint32_t *tickets;
    const void *x, *dt, *B, *C, *z;
    const float *conv_w, *conv_b, *A, *Dskip, *dt_bias;
    const int32_t *idx;
    void *y;
    int64_t n_slots, D, Bt;
    int W, delta_softplus;
};

// Shared-memory stage of one row: checkpoint block (fp32, or the bf16 copy in
// its first half), W-1 buffer entries of kCh (delta, delta*xc) pairs, the
// buffered tokens' B rows (fp32), conv state, x, dt, z. This token's B and C
// rows come from a per-batch fp32 table (below), so the replay loop and the
// readout read shared memory only.
template <typename T, typename TC, int K>
struct Stage {
    static constexpr uint32_t H = kCh * kN * 4;
    static constexpr uint32_t ENTRY = kCh * 8;
    static constexpr uint32_t BROW = kN * 4;  // one buffered B row (fp32)
    static constexpr uint32_t CS = (kCh * (K - 1) * sizeof(TC) + 15) / 16 * 16;
    static constexpr uint32_t AC = (kCh * sizeof(T) + 15) / 16 * 16;
    uint32_t off_bb, off_cs, off_x, off_dt, off_z, bytes;
    __host__ __device__ explicit Stage(int W)
    {
        off_bb = H + (uint32_t)(W - 1) * ENTRY;
        off_cs = off_bb + (uint32_t)(W - 1) * BROW;
        off_x = off_cs + CS;
        off_dt = off_x + AC;
        off_z = off_dt + AC;
        bytes = (off_z + AC + 127) / 128 * 128;
    }
};

// Rows whose slot, buffer length and fp32 B and C rows a CTA holds at once.
constexpr int kRowBatch = 32;

template <typename T, typename TC, int K>
size_t smem_bytes(int W)
{
    return (size_t)kStages * Stage<T, TC, K>(W).bytes + 16 * kStages +
           (size_t)kRowBatch * (8 + 2 * kN * 4);
}

// Four consecutive fp32 entries starting at a multiple of 4, as two packed pairs.
__device__ __forceinline__ void load4f(const float *p, f32x2 &lo, f32x2 &hi)
{
    const float4 v = __ldg(reinterpret_cast<const float4 *>(p));
    lo = pk2(v.x, v.y);
    hi = pk2(v.z, v.w);
}

// The same from shared memory.
__device__ __forceinline__ void lds4f(const float *p, f32x2 &lo, f32x2 &hi)
{
    const float4 v = *reinterpret_cast<const float4 *>(p);
    lo = pk2(v.x, v.y);
    hi = pk2(v.z, v.w);
}

// One token of the recurrence on four states held as two packed pairs:
// h = 2^(d * A log2 e) * h + u * B, with the operations and their order of the
// eager decode kernel.
__device__ __forceinline__ void token4(float4 &h4, f32x2 a01, f32x2 a23, f32x2 dd, f32x2 uu,
                                       f32x2 b01, f32x2 b23, f32x2 &h01, f32x2 &h23)
{
    float e0, e1, e2, e3;
    upk2(mul2(dd, a01), e0, e1);
    upk2(mul2(dd, a23), e2, e3);
    h01 = fma2(pk2(ex2_approx(e0), ex2_approx(e1)), pk2(h4.x, h4.y), mul2(uu, b01));
    h23 = fma2(pk2(ex2_approx(e2), ex2_approx(e3)), pk2(h4.z, h4.w), mul2(uu, b23));
    upk2(h01, h4.x, h4.y);
    upk2(h23, h4.z, h4.w);
}

// The same on states held as two packed pairs h01, h23 (no unpacking).
__device__ __forceinline__ void token2(f32x2 &h01, f32x2 &h23, f32x2 a01, f32x2 a23, f32x2 dd,
                                       f32x2 uu, f32x2 b01, f32x2 b23)
{
    float e0, e1, e2, e3;
    upk2(mul2(dd, a01), e0, e1);
    upk2(mul2(dd, a23), e2, e3);
    h01 = fma2(pk2(ex2_approx(e0), ex2_approx(e1)), h01, mul2(uu, b01));
    h23 = fma2(pk2(ex2_approx(e2), ex2_approx(e3)), h23, mul2(uu, b23));
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// ---------------------------------------------------------------------------
// step kernel (all row slices 16-byte aligned; the host checks)
//
// Warp-specialised: kCh compute threads own one channel each (all 16 states
// in packed fp32x2 registers) and one producer warp moves the data. A CTA
// walks rows gridDim.y apart in batches of up to kRowBatch rows. For a batch,
// the compute threads first read every row's slot and buffer length and
// convert its B and C rows to fp32 into a shared table (once per CTA rather
// than once per thread). The producer then streams each row's other inputs
// into a shared-memory stage with 1-D bulk copies, kStages rows ahead; a
// stage's "full" barrier completes when its bytes land and its "done" barrier
// when the compute warps have finished it, after which the producer stores
// the updated conv state (and, on checkpoint steps, the fp32 checkpoint) from
// the stage and refills it. Within a batch the compute warps never wait for
// one another.
//
// Register vector q holds states 4m..4m+3 with m = (q + rot) mod 4 and
// rot = (t / 4) mod 4, so the 8-byte reads of the bf16 copy (16 lanes per
// shared-memory wavefront) hit 16 different bank pairs; A and the B and C
// rows are read in the same order.
// ---------------------------------------------------------------------------
constexpr int kComputeWarps = kCh / 32;
constexpr int kThreads = kCh + 32;  // compute warps, then the producer warp

template <typename T, typename TC, int K>
__global__ void __launch_bounds__(kThreads, 4)  // 4 CTAs per SM: at most 102 registers
replay_step_kernel(const RParams p)
{
    using G = Stage<T, TC, K>;
    const G g(p.W);
    extern __shared__ __align__(128) unsigned char smem[];
    // after the stages (128-byte aligned): the fp32 B and C table, read as
    // 16-byte vectors, then the stage barriers, then the row metadata
    float *row_bc = reinterpret_cast<float *>(smem + kStages * g.bytes);  // [row][B 16 | C 16]
    uint64_t *full = reinterpret_cast<uint64_t *>(row_bc + kRowBatch * 2 * kN);
    uint64_t *done = full + kStages;
    int *row_slot = reinterpret_cast<int *>(done + kStages);  // -1: row skipped
    int *row_len = row_slot + kRowBatch;
    const int t = threadIdx.x;
    const int64_t D = p.D, DN = p.D * kN;
    const int64_t c0 = (int64_t)blockIdx.x * kCh;
    const int nch = (int)min((int64_t)kCh, D - c0);
    const int64_t c = c0 + t;
    const bool cvalid = t < nch;
    const int64_t rstep = gridDim.y, r0 = blockIdx.y;
    const int nrows = (int)((p.Bt - r0 + rstep - 1) / rstep);
    const int W = p.W;
    const bool has_lo = p.ckpt_lo != nullptr;
    const bool has_z = p.z != nullptr;
    const uint32_t h32_b = (uint32_t)nch * kN * 4, h16_b = (uint32_t)nch * kN * 2;
    const uint32_t ent_b = (uint32_t)nch * 8;
    const uint32_t cs_b = (uint32_t)(nch * (K - 1) * sizeof(TC));
    const uint32_t a_b = (uint32_t)(nch * sizeof(T));
    const uint32_t io_b = (uint32_t)(has_z ? 3 : 2) * a_b;
    TC *CS = static_cast<TC *>(p.conv_state);
    const T *X = static_cast<const T *>(p.x);
    const T *DT = static_cast<const T *>(p.dt);
    const T *Z = static_cast<const T *>(p.z);
    const T *Bg = static_cast<const T *>(p.B);
    const T *Cg = static_cast<const T *>(p.C);
    bool failed = false;

    if (t == kCh) {
        for (int st = 0; st < kStages; ++st) {
            mbar_init_n(&full[st], 1);
            mbar_init_n(&done[st], kComputeWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }

    if (t >= kCh) {
        // ------------------------------------------------------------------
        // producer warp: lane 0 moves the data; the other lanes only join the
        // batch barriers
        // ------------------------------------------------------------------
        const bool lead = t == kCh;
        int st = 0;
        uint32_t round = 0;     // completed passes over the stages
        uint32_t held = 0;      // bit i: stage i holds a row that is not stored yet
        uint32_t held_ph = 0;   // bit i: parity of that row's "done" phase
        int pend_slot[kStages];
        bool pend_flush[kStages];
#pragma unroll
        for (int i = 0; i < kStages; ++i) {
            pend_slot[i] = -1;
            pend_flush[i] = false;
        }
        // wait until the compute warps are done with stage i, then store its
        // conv state (and checkpoint) from it
        auto retire = [&](int i) {
            mbar_wait(&done[i], (held_ph >> i) & 1u, failed, &g_replay_status, 1);
            const int64_t sl = pend_slot[i];
            if (sl >= 0) {
                const unsigned char *sp = smem + (size_t)i * g.bytes;
                if (pend_flush[i]) bulk_s2g(p.ckpt + sl * DN + c0 * kN, sp, h32_b);
                bulk_s2g(CS + (sl * D + c0) * (K - 1), sp + g.off_cs, cs_b);
            }
            bulk_commit();
            held &= ~(1u << i);
        };
        // the channel block's offsets, folded in once; the row's activations
        // advance by rstep rows per row
        const float *ck_c = p.ckpt + c0 * kN;
        const __nv_bfloat16 *lo_c = p.ckpt_lo + c0 * kN;
        const float *buf_c = p.buf + c0 * 2;
        TC *cs_c = CS + c0 * (K - 1);
        const int64_t wd = (int64_t)(W - 1) * D * 2;  // one slot's buffer, in floats
        int64_t xoff = r0 * D + c0;
        const int64_t xstep = rstep * D;
        for (int b0 = 0; b0 < nrows; b0 += kRowBatch) {
            const int nb = min(kRowBatch, nrows - b0);
            __syncthreads();  // the batch's metadata and B/C table are ready
            if (lead) {
                for (int jj = 0; jj < nb; ++jj, xoff += xstep) {
                    if (held & (1u << st)) {
                        retire(st);
                        bulk_wait_read<0>();  // the stores have read the stage
                    }
                    const int64_t s = row_slot[jj];
                    held |= 1u << st;
                    held_ph = (held_ph & ~(1u << st)) | ((round & 1u) << st);
                    pend_slot[st] = (int)s;
                    pend_flush[st] = false;
                    if (s < 0) {
                        mbar_arrive(&full[st]);  // row skipped: complete the phase without data
                    } else {
                        const int jl = row_len[jj];
                        const bool flush = jl + 1 == W;
                        pend_flush[st] = flush;
                        unsigned char *dst = smem + (size_t)st * g.bytes;
                        const uint32_t hb = (flush || !has_lo) ? h32_b : h16_b;
                        mbar_expect_tx(&full[st],
                                       hb + (uint32_t)jl * (ent_b + G::BROW) + cs_b + io_b);
                        if (flush || !has_lo)
                            bulk_g2s(dst, ck_c + s * DN, hb, &full[st]);
                        else
                            bulk_g2s(dst, lo_c + s * DN, hb, &full[st]);
                        const float *bsrc = buf_c + s * wd;
                        for (int i = 0; i < jl; ++i)
                            bulk_g2s(dst + G::H + (uint32_t)i * G::ENTRY,
                                     bsrc + (int64_t)i * D * 2, ent_b, &full[st]);
                        if (jl > 0)
                            bulk_g2s(dst + g.off_bb, p.bufB + s * (int64_t)(W - 1) * kN,
                                     (uint32_t)jl * G::BROW, &full[st]);
                        bulk_g2s(dst + g.off_cs, cs_c + s * D * (K - 1), cs_b, &full[st]);
                        bulk_g2s(dst + g.off_x, X + xoff, a_b, &full[st]);
                        bulk_g2s(dst + g.off_dt, DT + xoff, a_b, &full[st]);
                        if (has_z) bulk_g2s(dst + g.off_z, Z + xoff, a_b, &full[st]);
                    }
                    if (++st == kStages) {
                        st = 0;
                        ++round;
                    }
                }
                // store the batch's last rows before the stages are reused
                for (int i = 0; i < kStages; ++i)
                    if (held & (1u << i)) retire(i);
                bulk_wait_read<0>();
            }
            __syncthreads();  // the compute warps take their tickets after this
            __syncthreads();  // the batch's table and metadata are no longer read
        }
        if (lead) bulk_wait<0>();
        return;
    }

    // ----------------------------------------------------------------------
    // compute warps
    // ----------------------------------------------------------------------
    float2 *buf_t = reinterpret_cast<float2 *>(p.buf) + c;
    __nv_bfloat16 *lo_t = p.ckpt_lo + c * kN;
    T *y_t = static_cast<T *>(p.y) + c;

    // per-channel parameters in the rotated order; A pre-scaled by log2(e)
    const int rot = (t >> 2) & 3;
    f32x2 A2[8];
    float w[K], cb = 0.f, dtb = 0.f, dsk = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int m = (q + rot) & 3;
        const float4 a4 = cvalid ? __ldg(reinterpret_cast<const float4 *>(p.A + c * kN + 4 * m))
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
        A2[2 * q] = pk2(a4.x * kLog2e, a4.y * kLog2e);
        A2[2 * q + 1] = pk2(a4.z * kLog2e, a4.w * kLog2e);
    }
#pragma unroll
    for (int k = 0; k < K; ++k) w[k] = cvalid ? __ldg(p.conv_w + c * K + k) : 0.f;
    if (cvalid) {
        cb = p.conv_b ? __ldg(p.conv_b + c) : 0.f;
        dtb = p.dt_bias ? __ldg(p.dt_bias + c) : 0.f;
        dsk = p.Dskip ? __ldg(p.Dskip + c) : 0.f;
    }

    int cons_st = 0;
    uint32_t cons_ph = 0;
    unsigned char *sp_cur = smem;  // the stage of cons_st
    T *yrow = y_t + r0 * D;        // this thread's y entry of the current row
    const int64_t ystep = rstep * D;
    for (int b0 = 0; b0 < nrows; b0 += kRowBatch) {
        const int nb = min(kRowBatch, nrows - b0);
        // Every row's slot and length are read once, in parallel, before any
        // of the batch's loads are issued; the lengths are advanced only after
        // the whole batch (tickets below), so each CTA reads them before it
        // takes a ticket.
        if (t < nb) {
            const int64_t b = r0 + (int64_t)(b0 + t) * rstep;
            int64_t sl = p.idx ? (int64_t)p.idx[b] : b;
            sl = (sl >= 0 && sl < p.n_slots) ? sl : -1;
            int jl = 0;
            if (sl >= 0) {
                jl = p.len[sl];
                jl = jl < 0 ? 0 : (jl > W - 1 ? W - 1 : jl);  // a corrupt length stays in bounds
            }
            row_slot[t] = (int)sl;
            row_len[t] = jl;
        }
        for (int e = t; e < nb * 2 * kN; e += kCh) {
            const int r = e / (2 * kN), k = e % (2 * kN);
            const int64_t b = r0 + (int64_t)(b0 + r) * rstep;
            row_bc[e] = to_f32(k < kN ? Bg[b * kN + k] : Cg[b * kN + (k - kN)]);
        }
        __syncthreads();

        for (int jj = 0; jj < nb; ++jj, yrow += ystep) {
            const int st = cons_st;
            mbar_wait(&full[st], cons_ph, failed, &g_replay_status, 1);
            const int64_t s = row_slot[jj];
            const int jl = row_len[jj];
            const bool flush = s >= 0 && jl + 1 == W;
            unsigned char *sp = sp_cur;
            if (s >= 0 && cvalid) {
                // the checkpoint: fp32, or the bf16 copy on the other steps
                f32x2 h2[8];
                if (flush || !has_lo) {
                    const float4 *sh = reinterpret_cast<const float4 *>(sp) + t * 4;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 v = sh[(q + rot) & 3];
                        h2[2 * q] = pk2(v.x, v.y);
                        h2[2 * q + 1] = pk2(v.z, v.w);
                    }
                } else {
                    const uint2 *sh = reinterpret_cast<const uint2 *>(sp) + t * 4;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint2 u = sh[(q + rot) & 3];
                        h2[2 * q] = pk2(bf16_lo(u.x), bf16_hi(u.x));
                        h2[2 * q + 1] = pk2(bf16_lo(u.y), bf16_hi(u.y));
                    }
                }
                // replay the buffered tokens, oldest first
                const float2 *ent = reinterpret_cast<const float2 *>(sp + G::H) + t;
                const float *bB = reinterpret_cast<const float *>(sp + g.off_bb);
                for (int i = 0; i < jl; ++i) {
                    const float2 du = ent[i * kCh];
                    const f32x2 dd = pk2(du.x, du.x), uu = pk2(du.y, du.y);
                    const float *bi = bB + i * kN;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        f32x2 b01, b23;
                        lds4f(bi + 4 * ((q + rot) & 3), b01, b23);
                        token2(h2[2 * q], h2[2 * q + 1], A2[2 * q], A2[2 * q + 1], dd, uu, b01,
                               b23);
                    }
                }
                // this token: conv, softplus, update and readout as in eager decode
                TC *scs = reinterpret_cast<TC *>(sp + g.off_cs) + t * (K - 1);
                float win[K];
#pragma unroll
                for (int k = 0; k < K - 1; ++k) win[k] = to_f32(scs[k]);
                win[K - 1] = to_f32(reinterpret_cast<const T *>(sp + g.off_x)[t]);
                float d = to_f32(reinterpret_cast<const T *>(sp + g.off_dt)[t]) + dtb;
                float acc = cb;
#pragma unroll
                for (int k = 0; k < K; ++k) acc = fmaf(w[k], win[k], acc);
                const float xcv = silu_f(acc);
                if (p.delta_softplus) d = softplus_fast(d);
                const float dx = d * xcv;
                const f32x2 dd = pk2(d, d), xx = pk2(dx, dx);
                const float *bc = row_bc + jj * 2 * kN;
                f32x2 yacc = 0ull;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int m = (q + rot) & 3;
                    f32x2 b01, b23, c01, c23;
                    lds4f(bc + 4 * m, b01, b23);
                    lds4f(bc + kN + 4 * m, c01, c23);
                    token2(h2[2 * q], h2[2 * q + 1], A2[2 * q], A2[2 * q + 1], dd, xx, b01, b23);
                    yacc = fma2(c01, h2[2 * q], yacc);
                    yacc = fma2(c23, h2[2 * q + 1], yacc);
                }
                if (flush) {
                    // new checkpoint: fp32 block back into the stage (the
                    // producer stores it), bf16 copy straight to global memory
                    float4 *sh = reinterpret_cast<float4 *>(sp) + t * 4;
                    uint32_t o[8];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int m = (q + rot) & 3;
                        float a0, a1, a2, a3;
                        upk2(h2[2 * q], a0, a1);
                        upk2(h2[2 * q + 1], a2, a3);
                        sh[m] = make_float4(a0, a1, a2, a3);
                        o[2 * q] = pack_bf16(a0, a1);
                        o[2 * q + 1] = pack_bf16(a2, a3);
                    }
                    if (has_lo) {
                        uint2 *lo = reinterpret_cast<uint2 *>(lo_t + s * DN);
#pragma unroll
                        for (int q = 0; q < 4; ++q) lo[(q + rot) & 3] = make_uint2(o[2 * q], o[2 * q + 1]);
                    }
                } else {
                    // buffer this token's SSM inputs
                    buf_t[(s * (W - 1) + jl) * D] = make_float2(d, dx);
                }
#pragma unroll
                for (int k = 0; k < K - 1; ++k) scs[k] = from_f32<TC>(win[k + 1]);
                float y0, y1;
                upk2(yacc, y0, y1);
                float yv = y0 + y1 + dsk * xcv;
                if (has_z) yv *= silu_f(to_f32(reinterpret_cast<const T *>(sp + g.off_z)[t]));
                *yrow = from_f32<T>(yv);
            }
            // the row's B joins the buffer once (channel block 0)
            if (s >= 0 && !flush && blockIdx.x == 0 && t < kN)
                p.bufB[(s * (W - 1) + jl) * kN + t] = row_bc[jj * 2 * kN + t];
            // this thread's shared-memory writes, before the producer's bulk stores read them
            fence_proxy_async();
            __syncwarp();
            if ((t & 31) == 0) mbar_arrive(&done[st]);
            sp_cur += g.bytes;
            if (++cons_st == kStages) {
                cons_st = 0;
                cons_ph ^= 1u;
                sp_cur = smem;
            }
        }
        // The last channel block of a row to finish advances its length: one
        // ticket per row and CTA, taken after this CTA read every length of
        // the batch (the fence orders that read before the ticket).
        __syncthreads();  // with the producer: every row of the batch is stored or queued
        if (t < nb && row_slot[t] >= 0) {
            const int sl = row_slot[t];
            __threadfence();
            const uint32_t prev = atomicAdd(&p.tickets[sl], 1u);
            if (prev == gridDim.x - 1) {
                p.len[sl] = (row_len[t] + 1 == W) ? 0 : row_len[t] + 1;
                p.tickets[sl] = 0;
            }
        }
        __syncthreads();  // the batch's table and metadata are no longer read
    }
}

// ---------------------------------------------------------------------------
// reset: start each listed slot's window at the state held in its checkpoint
// ---------------------------------------------------------------------------
__global__ void replay_reset_kernel(const float *ckpt, __nv_bfloat16 *ckpt_lo, int32_t *len,
                                    uint32_t *tickets, const int32_t *slots, int64_t n,
                                    int64_t n_slots, int64_t D)
{
    const int64_t i = (int64_t)blockIdx.y;
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int64_t s = slots ? (int64_t)slots[i] : i;
    if (s < 0 || s >= n_slots) return;
    if (c == 0) {
        len[s] = 0;
        tickets[s] = 0;
    }
    if (c >= D || ckpt_lo == nullptr) return;
    const float4 *h = reinterpret_cast<const float4 *>(ckpt + (s * D + c) * kN);
    float4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = h[q];
    uint4 o0, o1;
    o0.x = pack_bf16(v[0].x, v[0].y); o0.y = pack_bf16(v[0].z, v[0].w);
    o0.z = pack_bf16(v[1].x, v[1].y); o0.w = pack_bf16(v[1].z, v[1].w);
    o1.x = pack_bf16(v[2].x, v[2].y); o1.y = pack_bf16(v[2].z, v[2].w);
    o1.z = pack_bf16(v[3].x, v[3].y); o1.w = pack_bf16(v[3].z, v[3].w);
    uint4 *lo = reinterpret_cast<uint4 *>(ckpt_lo + (s * D + c) * kN);
    lo[0] = o0;
    lo[1] = o1;
}

// ---------------------------------------------------------------------------
// flush: replay every buffered token into the fp32 checkpoint and refresh the
// bf16 copy (the lengths are cleared by a second launch, after every channel
// has read them)
// ---------------------------------------------------------------------------
__global__ void replay_flush_kernel(float *ckpt, __nv_bfloat16 *ckpt_lo, const float *buf,
                                    const float *bufB, const int32_t *len, const float *A, int W,
                                    const int32_t *slots, int64_t n, int64_t n_slots, int64_t D)
{
    const int64_t i = (int64_t)blockIdx.y;
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n || c >= D) return;
    const int64_t s = slots ? (int64_t)slots[i] : i;
    if (s < 0 || s >= n_slots) return;
    int jl = len[s];
    jl = jl < 0 ? 0 : (jl > W - 1 ? W - 1 : jl);
    float4 *hp = reinterpret_cast<float4 *>(ckpt + (s * D + c) * kN);
    float4 hq[4];
    f32x2 A2[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        hq[q] = hp[q];
        const float4 a4 = __ldg(reinterpret_cast<const float4 *>(A + c * kN + 4 * q));
        A2[2 * q] = pk2(a4.x * kLog2e, a4.y * kLog2e);
        A2[2 * q + 1] = pk2(a4.z * kLog2e, a4.w * kLog2e);
    }
    for (int e = 0; e < jl; ++e) {
        const float2 du = reinterpret_cast<const float2 *>(buf)[((s * (W - 1) + e) * D) + c];
        const f32x2 dd = pk2(du.x, du.x), uu = pk2(du.y, du.y);
        const float *bB = bufB + (s * (W - 1) + e) * kN;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            f32x2 b01, b23, h01, h23;
            load4f(bB + 4 * q, b01, b23);
            token4(hq[q], A2[2 * q], A2[2 * q + 1], dd, uu, b01, b23, h01, h23);
        }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) hp[q] = hq[q];
    if (ckpt_lo) {
        uint4 o0, o1;
        o0.x = pack_bf16(hq[0].x, hq[0].y); o0.y = pack_bf16(hq[0].z, hq[0].w);
        o0.z = pack_bf16(hq[1].x, hq[1].y); o0.w = pack_bf16(hq[1].z, hq[1].w);
        o1.x = pack_bf16(hq[2].x, hq[2].y); o1.y = pack_bf16(hq[2].z, hq[2].w);
        o1.z = pack_bf16(hq[3].x, hq[3].y); o1.w = pack_bf16(hq[3].z, hq[3].w);
        uint4 *lo = reinterpret_cast<uint4 *>(ckpt_lo + (s * D + c) * kN);
        lo[0] = o0;
        lo[1] = o1;
    }
}

__global__ void replay_clear_len_kernel(int32_t *len, uint32_t *tickets, const int32_t *slots,
                                        int64_t n, int64_t n_slots)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int64_t s = slots ? (int64_t)slots[i] : i;
    if (s < 0 || s >= n_slots) return;
    len[s] = 0;
    tickets[s] = 0;
}

template <typename T, typename TC, int K>
cudaError_t run_step(const RParams &p, cudaStream_t stream, int *launches)
{
    const size_t smem = smem_bytes<T, TC, K>(p.W);
    cudaError_t e = cudaFuncSetAttribute(replay_step_kernel<T, TC, K>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, replay_step_kernel<T, TC, K>, kThreads,
                                                      smem) != cudaSuccess)
        return cudaErrorUnknown;
    const int64_t gx = (p.D + kCh - 1) / kCh;
    int64_t gy = ((int64_t)sms * (per_sm > 0 ? per_sm : 1)) / gx;
    gy = gy < 1 ? 1 : (gy > p.Bt ? p.Bt : gy);
    if (gy > 65535) gy = 65535;
    replay_step_kernel<T, TC, K><<<dim3((unsigned)gx, (unsigned)gy), kThreads, smem, stream>>>(p);
    ++*launches;
    return cudaGetLastError();
}

template <typename T, typename TC>
cudaError_t by_k(const RParams &p, int K, cudaStream_t s, int *n)
{
    switch (K) {
    case 2: return run_step<T, TC, 2>(p, s, n);
    case 3: return run_step<T, TC, 3>(p, s, n);
    default: return run_step<T, TC, 4>(p, s, n);
    }
}

}  // namespace

struct ReplayStepArgs {
    void *conv_state;
    float *ckpt;
    void *ckpt_lo;
    float *buf, *bufB;
    int32_t *len;
    uint32_t *tickets;
    int W;
    const void *x, *dt, *B, *C, *z;
    const float *conv_w, *conv_b, *A, *Dskip, *dt_bias;
    int delta_softplus;
    const int32_t *idx;
    int64_t n_slots;
    void *y;
    int64_t Bt, D;
    int K;
    bool act_bf16, conv_bf16;
};

cudaError_t launch_replay_step(const ReplayStepArgs &a, cudaStream_t stream, int *launches)
{
    if (a.Bt == 0) return cudaSuccess;
    RParams p;
    p.conv_state = a.conv_state; p.ckpt = a.ckpt;
    p.ckpt_lo = static_cast<__nv_bfloat16 *>(a.ckpt_lo);
    p.buf = a.buf; p.bufB = a.bufB; p.len = a.len; p.tickets = a.tickets;
    p.x = a.x; p.dt = a.dt; p.B = a.B; p.C = a.C; p.z = a.z;
    p.conv_w = a.conv_w; p.conv_b = a.conv_b; p.A = a.A; p.Dskip = a.Dskip;
    p.dt_bias = a.dt_bias; p.idx = a.idx; p.y = a.y;
    p.n_slots = a.n_slots; p.D = a.D; p.Bt = a.Bt; p.W = a.W;
    p.delta_softplus = a.delta_softplus;
    if (a.act_bf16 && a.conv_bf16) return by_k<__nv_bfloat16, __nv_bfloat16>(p, a.K, stream, launches);
    if (a.act_bf16) return by_k<__nv_bfloat16, float>(p, a.K, stream, launches);
    if (a.conv_bf16) return by_k<float, __nv_bfloat16>(p, a.K, stream, launches);
    return by_k<float, float>(p, a.K, stream, launches);
}

cudaError_t launch_replay_reset(const float *ckpt, void *ckpt_lo, int32_t *len, uint32_t *tickets,
                                const int32_t *slots, int64_t n, int64_t n_slots, int64_t D,
                                cudaStream_t stream, int *launches)
{
    if (n == 0) return cudaSuccess;
    const dim3 grid((unsigned)((D + 127) / 128), (unsigned)n);
    replay_reset_kernel<<<grid, 128, 0, stream>>>(ckpt, static_cast<__nv_bfloat16 *>(ckpt_lo),
                                                  len, tickets, slots, n, n_slots, D);
    ++*launches;
    return cudaGetLastError();
}

cudaError_t launch_replay_flush(float *ckpt, void *ckpt_lo, const float *buf, const float *bufB,
                                int32_t *len, uint32_t *tickets, const float *A, int W,
                                const int32_t *slots, int64_t n, int64_t n_slots, int64_t D,
                                cudaStream_t stream, int *launches)
{
    if (n == 0) return cudaSuccess;
    const dim3 grid((unsigned)((D + 127) / 128), (unsigned)n);
    replay_flush_kernel<<<grid, 128, 0, stream>>>(ckpt, static_cast<__nv_bfloat16 *>(ckpt_lo),
                                                  buf, bufB, len, A, W, slots, n, n_slots, D);
    ++*launches;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    replay_clear_len_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(len, tickets, slots,
                                                                            n, n_slots);
    ++*launches;
    return cudaGetLastError();
}

int read_replay_status(bool clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_replay_status, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_replay_status, &zero, sizeof(int)) != cudaSuccess) return -1;
    }
    return v;
}

}  // namespace ssm
