/*
 * csa2.h — C ABI of libcsa2: the CSA2 decode step over a globally cached FP4 KV,
 * hand-written CUDA for sm_100a (B200).
 *
 * Sources (web pages describing the DeepSeek-V4.1-Flash technical report):
 *   P1 = onedev.kr, "KV 캐시를 토큰당 890바이트로 압축한 552B 멀티모달 MoE, DeepSeek-V4.1-Flash"
 *   P2 = thakicloud tech blog, "DeepSeek V4.1-Flash KV compression"
 *   P3 = genexis.ai, "100만 토큰을 0.9GB에, 딥시크 V4.1 논문이 KV 캐시를 줄인 방법"
 * A citation reads "P3 §<section heading>".
 *
 * Conventions shared by every entry point
 *  - Every pointer argument is a DEVICE pointer owned by the caller (except the string
 *    returned by csa2_status_string).  The library allocates nothing, keeps no pointer
 *    after returning, holds no global mutable state and never synchronises: each call
 *    validates its host-visible arguments, enqueues its kernels on `stream` and returns.
 *    The one exception is csa2_reindex_static (end of this file), which uses a device
 *    array compiled into the library and caches its address per device context.
 *  - On CSA2_ERR_INVALID_ARG or CSA2_ERR_UNSUPPORTED nothing has been launched.
 *    CSA2_ERR_CUDA reports a launch failure (cudaGetLastError after the launch).
 *  - Values that live on the device (sequence bases, visible counts, Top-K indices,
 *    block ids, destination entries) are range-checked by the kernels: an offending
 *    item is skipped (treated as empty) and a bit is OR-ed into `*dev_status` (a device
 *    uint32, may be NULL); csa2_status_from_device_word() maps the word to a status.
 *  - Scratch ("workspace") is caller-allocated device memory of at least the size the
 *    matching *_workspace_size() function returns; its contents need no initialisation
 *    and are garbage afterwards.  Base alignment: 256 bytes.
 *  - Layouts are dense row-major in the order written [a][b][c].  Required base
 *    alignment: 16 bytes for every array except the int32/int64 index arrays (4/8).
 *  - Inputs must be finite; entries, scores and outputs derived from NaN/Inf inputs
 *    are unspecified.
 *
 * Data structures (P3 §레이어 40개 가운데 4개만 전역 캐시를 만듭니다, §4비트로 적어도
 * 되는 이유; P2 §KV 캐시 네 가지):
 *  - KV entry, 288 bytes: a 512-channel latent in E2M1 (4-bit) with one E4M3 scale per
 *    16 channels and no second-level scale.  Byte i (0..255) holds channel 2i in its low
 *    nibble and channel 2i+1 in its high nibble; byte 256+b is the scale of channels
 *    16b..16b+15.  Value = E4M3(scale) * E2M1(code).
 *  - Indexer-key entry, 68 bytes: 128 dims of E2M1 codes (bytes 0..63, same nibble
 *    order) then one little-endian fp32 scale (bytes 64..67).  Value = scale * E2M1.
 *  - A pool is an array of entries; sequence b owns entries seq_base[b] + j, j >= 0.
 *  - Sliding window: E4M3 bytes [B][S_w][512]; row r of sequence b is token
 *    swa_start[b] + r.  The query at token t sees tokens max(0, t-window+1)..t that lie
 *    in its sequence's buffer (P3 §전역 어텐션과 지역 어텐션: a 128-token window).
 *  - Causal visibility is a prefix: query (b,i) sees entries [0, n_vis[b*Q+i]).
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CSA2_D 512               /* main-KV latent channels */
#define CSA2_DI 128              /* indexer-key dimension */
#define CSA2_KV_ENTRY_BYTES 288  /* 256 B codes + 32 B E4M3 scales */
#define CSA2_IK_ENTRY_BYTES 68   /* 64 B codes + 4 B fp32 scale */
#define CSA2_MAX_K 2048          /* largest Top-K / block count per query */
#define CSA2_MAX_HI 16           /* largest number of indexer heads */
#define CSA2_MAX_WINDOW 1024     /* largest sliding window */
#define CSA2_STATIC_SCRATCH_BYTES (4u << 20) /* device array behind csa2_reindex_static */
#define CSA2_MAX_SHARDS 64       /* largest number of context-parallel shards per merge */

typedef enum csa2_status {
  CSA2_OK = 0,
  CSA2_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size; nothing launched */
  CSA2_ERR_UNSUPPORTED = 2,  /* valid request outside the supported shapes */
  CSA2_ERR_CUDA = 3,         /* a kernel launch failed */
  CSA2_ERR_TIMEOUT = 4,      /* a device-side wait hit its iteration cap */
  CSA2_ERR_DEVICE_INPUT = 5  /* a kernel found an out-of-range device-side value */
} csa2_status;

/* Bits of the device status word. */
#define CSA2_DEV_BAD_INDEX 0x1u  /* entry/block index or destination out of range */
#define CSA2_DEV_BAD_COUNT 0x2u  /* n_vis outside [0, max_n_vis] or past the pool */
#define CSA2_DEV_TIMEOUT 0x4u    /* bounded wait expired */

const char* csa2_status_string(csa2_status s);
/* Map a device status word (OR of CSA2_DEV_* bits) to a status; 0 -> CSA2_OK. */
csa2_status csa2_status_from_device_word(uint32_t word);
/* Library version: major*10000 + minor*100 + patch. */
int csa2_version(void);

/* ---------------------------------------------------------------------------------
 * a1  Pack new global-KV entries (P3 §레이어 40개 가운데 4개만 전역 캐시를 만듭니다:
 * 288 B main KV + 68 B indexer key per entry; encoder Full layers store one entry per
 * 2 tokens, the decoder Full layer one per token; P3 §4비트로 적어도 되는 이유: NVFP4
 * without the global scale, one 8-bit scale per 16 channels).
 *
 *   kv   bf16 [T][512]   raw main-KV tokens (already normalised/rotated by the model)
 *   ik   bf16 [T][128]   raw indexer-key tokens
 *   T    tokens; ratio 1 (one entry per token) or 2 (one per token pair; T even)
 *   dst_entry  int64 [T/ratio]: pool slot of each new entry, or NULL for slots 0..T/ratio-1
 *   pool_entries  number of entries the two pools hold (destinations are checked)
 *   kv_pool  u8 [pool_entries][288], ik_pool u8 [pool_entries][68]: written in place
 *
 * Per entry (ratio 2: every channel is first replaced by the fp32 mean (a+b)*0.5f of
 * the token pair):
 *   main KV, per 16-channel block: amax = max|x|; s = E4M3_RNE_sat(amax/6 in fp32);
 *     code = E2M1_RNE_sat(x / value(s)) with the quotient rounded to fp32, ties to the
 *     even code, sign kept on zero; value(s) == 0 gives +0 codes.
 *   indexer key: s = amax/6 (fp32, stored); code = E2M1_RNE_sat(x / s); s == 0 -> +0.
 * Output is bit-exact with that definition.  Destinations outside [0, pool_entries)
 * are skipped and flag CSA2_DEV_BAD_INDEX.
 * --------------------------------------------------------------------------------- */
csa2_status csa2_pack_kv(const void* kv, const void* ik, int64_t T, int ratio,
                         const int64_t* dst_entry, int64_t pool_entries, uint8_t* kv_pool,
                         uint8_t* ik_pool, uint32_t* dev_status, cudaStream_t stream);

/* ---------------------------------------------------------------------------------
 * a1 producer: RMSNorm + rotary encoding + pack (P3 §4비트로 적어도 되는 이유: cached
 * values are normalised and rotated before caching, which bounds them by sqrt(512);
 * the pages give no formula, so the operations below are this library's reading).
 *
 *   kv   bf16 [T][512]  raw (not yet normalised) main-KV tokens
 *   ik   bf16 [T][128]  indexer-key tokens (packed as csa2_pack_kv packs them)
 *   pos  int64 [T]      row of the rotation tables for each token (its position)
 *   rope_cos, rope_sin  fp32 [n_pos][256]: cosine and sine for channel pair i at each row
 *   gamma fp32 [512] per-channel gain, or NULL for none;  eps >= 0
 *   T, ratio, dst_entry, pool_entries, kv_pool, ik_pool: as csa2_pack_kv
 *
 * Per token, every operation rounded once in fp32 (no fused multiply-add):
 *   S = sum of x_c^2, summed by halving within each 16-channel block (element i += i+8,
 *       then +4, +2, +1), then by halving over the 32 block sums (+16, +8, +4, +2, +1);
 *   r = 1 / sqrt(S / 512 + eps) (the add, the square root and the reciprocal each
 *       correctly rounded);  n_c = x_c * r, then n_c * gamma_c;
 *   channel pairs (2i, 2i+1) rotated with c = rope_cos[pos][i], s = rope_sin[pos][i]:
 *       y_2i = n_2i c - n_2i+1 s,  y_2i+1 = n_2i s + n_2i+1 c;
 *   y rounded to bf16 (nearest, ties to even), then encoded exactly as csa2_pack_kv
 *   encodes a bf16 token (ratio 2: each token at its own position, then the pair mean).
 * Output is bit-exact with that definition.  An entry whose destination or either
 * position is out of range is skipped and flags CSA2_DEV_BAD_INDEX.
 * --------------------------------------------------------------------------------- */
csa2_status csa2_pack_kv_normed(const void* kv, const void* ik, int64_t T, int ratio, const int64_t* pos,
                                const float* rope_cos, const float* rope_sin, int64_t n_pos,
                                const float* gamma, float eps, const int64_t* dst_entry,
                                int64_t pool_entries, uint8_t* kv_pool, uint8_t* ik_pool,
                                uint32_t* dev_status, cudaStream_t stream);

/* ---------------------------------------------------------------------------------
 * a2+a3  Full-mode indexer scan with flat Top-K (P1 §무엇과 다른가: a Full layer scores
 * the whole causally visible range with its own indexer Q and picks Top-K).
 *
 *   q    fp32 [B][Q][HI][128]  indexer queries;  w  fp32 [B][Q][HI]  head weights
 *   ik_pool u8 [pool_entries][68];  seq_base int64 [B];  n_vis int32 [B][Q]
 *   max_n_vis  host-side upper bound on every n_vis (sizes the grid and workspace),
 *              at most 2^23
 *   topk int32 [B][Q][K]  out: the K best visible entries (indices relative to
 *        seq_base), -1 in unused slots; topk_score fp32 [B][Q][K] (may be NULL)
 *
 * score_j = sum_h w_h * max(0, q_h . k_j) over dequantised keys k_j.  Arithmetic: each
 * query head is scaled by a power of two and split into two f16 parts, hi + lo, which
 * represent it to 2^-22 of each element; the key's E2M1 values are exact in f16; the
 * tensor cores form every product exactly and sum both parts' products in fp32; fp32 then
 * applies the ReLU, the head weights and the key's scale.  The result is a SET
 * (slot order unspecified); equal scores at the cut prefer lower indices.
 * 1 <= K <= 2048, 1 <= HI <= 16.
 * --------------------------------------------------------------------------------- */
size_t csa2_index_full_workspace_size(int B, int Q, int HI, int K, int64_t max_n_vis);
csa2_status csa2_index_full(const float* q, const float* w, const uint8_t* ik_pool,
                            int64_t pool_entries, const int64_t* seq_base, const int32_t* n_vis,
                            int B, int Q, int HI, int K, int64_t max_n_vis, int32_t* topk,
                            float* topk_score, void* ws, size_t ws_bytes, uint32_t* dev_status,
                            cudaStream_t stream);

/* ---------------------------------------------------------------------------------
 * a2+a4  Hierarchical block selection (P1 §무엇과 다른가; P3 §레이어 40개 가운데 4개만
 * 전역 캐시를 만듭니다: the decoder's first Full layer scans the whole context and
 * keeps up to 2,048 blocks of 8 positions, a 16,384-position candidate pool).
 *
 * Same inputs as csa2_index_full.  Block c of a query holds its visible entries
 * [block*c, block*c+block); its score is the max of their scores.  blocks int32
 * [B][Q][n_blocks] receives the n_blocks best block ids (a set, -1 in unused slots);
 * block_score fp32 [B][Q][n_blocks] may be NULL.  1 <= n_blocks <= 2048;
 * block in {1,2,4,8,16,32}.
 * --------------------------------------------------------------------------------- */
size_t csa2_index_hier_workspace_size(int B, int Q, int HI, int n_blocks, int block,
                                      int64_t max_n_vis);
csa2_status csa2_index_hier(const float* q, const float* w, const uint8_t* ik_pool,
                            int64_t pool_entries, const int64_t* seq_base, const int32_t* n_vis,
                            int B, int Q, int HI, int n_blocks, int block, int64_t max_n_vis,
                            int32_t* blocks, float* block_score, void* ws, size_t ws_bytes,
                            uint32_t* dev_status, cudaStream_t stream);

/* ---------------------------------------------------------------------------------
 * a5  Reindex (P1 §무엇과 다른가: a Reindex layer reuses an earlier layer's cache and
 * rescoring with its own indexer Q picks a new Top-K; P3 §레이어 40개 가운데 4개만 전역
 * 캐시를 만듭니다: Reindex layers pick 512 inside the block pool).
 *
 * blocks int32 [B][Q][n_blocks] (from csa2_index_hier; ids distinct, -1 = empty).  The
 * candidates are the visible entries of those blocks; the result is the Top-K of them
 * by the layer's own q/w, under csa2_index_full's score and tie rule.  Arithmetic: each
 * query head is split into four int8 limbs (to 2^-22 of its largest element), the dot
 * products with the codes are exact int32 sums on the tensor cores and fp32 combines the
 * limbs (a K = 32 MMA step keeps this one-tile-per-CTA kernel's chain short).  Block ids
 * past the pool are skipped and flag CSA2_DEV_BAD_INDEX.
 * --------------------------------------------------------------------------------- */
size_t csa2_reindex_workspace_size(int B, int Q, int HI, int n_blocks, int block, int K);
csa2_status csa2_reindex(const float* q, const float* w, const uint8_t* ik_pool,
                         int64_t pool_entries, const int64_t* seq_base, const int32_t* n_vis,
                         const int32_t* blocks, int n_blocks, int block, int B, int Q, int HI,
                         int K, int32_t* topk, float* topk_score, void* ws, size_t ws_bytes,
                         uint32_t* dev_status, cudaStream_t stream);

/* ---------------------------------------------------------------------------------
 * a6+a7  Sparse MQA attention over Top-K FP4 entries plus the FP8 window (P1 §어떻게
 * 동작하나: a global branch plus sliding-window attention in every CSA2 layer; P3
 * §전역 어텐션과 지역 어텐션: a 128-token window; P3 §4비트로 적어도 되는 이유: the
 * window stays in 8 bits; P1 §무엇과 다른가: a Reuse layer attends with the Top-K list
 * it inherits, so Reuse = this call with that list).
 *
 *   q     fp32 [B][Q][H][512]   all H heads of a query share one key set (MQA)
 *   kv_pool u8 [pool_entries][288]; seq_base int64 [B]
 *   topk  int32 [B][Q][K]   entry indices relative to seq_base, -1 = empty slot
 *   swa   u8 [B][S_w][512] E4M3 window tokens (NULL when S_w == 0)
 *   swa_start int64 [B]; q_pos int64 [B][Q] token position of each query; window <= 1024
 *   out   fp32 [B][Q][H][512];  lse fp32 [B][Q][H] (natural log)
 *
 * Keys = {dequant(entry j) : j in topk, j >= 0} U {window tokens}; key = value;
 * logit = sm_scale * q_h . k.  QK^T and PV run on the tcgen05 tensor cores with f16
 * operands and fp32 accumulation: dequantised entries (E2M1 x E4M3, at most 2688) and
 * E4M3 window tokens are exact in f16; queries (times sm_scale*log2 e) and softmax
 * probabilities are rounded to f16, so |q| * sm_scale must stay below 4e4.  An empty
 * key set gives out = 0, lse = -inf.  H in {16, 32, 48, 64}.
 * q is read while the previous library kernel in the stream may still be running (the
 * call's kernels are launched to overlap their predecessor's tail): it must not be an
 * output of a libcsa2 call, which no libcsa2 call ever produces.
 * --------------------------------------------------------------------------------- */
size_t csa2_sparse_attn_workspace_size(int B, int Q, int H, int K, int window);
csa2_status csa2_sparse_attn(const float* q, const uint8_t* kv_pool, int64_t pool_entries,
                             const int64_t* seq_base, const int32_t* topk, int K,
                             const uint8_t* swa, int S_w, const int64_t* swa_start,
                             const int64_t* q_pos, int window, int B, int Q, int H,
                             float sm_scale, float* out, float* lse, void* ws, size_t ws_bytes,
                             uint32_t* dev_status, cudaStream_t stream);

/* ---------------------------------------------------------------------------------
 * Context-parallel decode: one sequence's cached entries split over C GPUs (ranks).
 * The pages describe one device; this decomposition is the library's reading of how
 * the same results split (P1 §무엇과 다른가: a Full layer's Top-K is taken over every
 * entry its query sees; P3 §전역 어텐션과 지역 어텐션: one softmax over the selected
 * entries and the window).  Rank c holds entries [lo_c, lo_c + len_c) of each sequence
 * in its own pool; the shards of a sequence are disjoint, contiguous and ordered by rank
 * (lo_0 < lo_1 < ...).  One Full layer then runs, on every rank:
 *   1. csa2_cp_shard_vis: the visible count inside the shard;
 *   2. csa2_index_full (or csa2_index_hier with lo_c a multiple of the block) on the
 *      rank's pool: its own Top-K with scores;
 *   3. an all-gather of the (index, score) lists over the ranks (the caller's
 *      collective, e.g. NCCL): [C][B][Q][K] each;
 *   4. csa2_topk_merge: the global Top-K (exact: the Top-K of the whole is the Top-K of
 *      the union of the shards' Top-K lists);
 *   5. csa2_topk_localize: the rank's own entries of that list, in its pool's indices;
 *   6. csa2_sparse_attn on them (the window on one rank only): out_c and lse_c;
 *   7. an all-gather of (out_c, lse_c) and csa2_attn_combine: attention over the union.
 * The library does not communicate; every call below is rank-local.
 * --------------------------------------------------------------------------------- */

/* n_vis_local[b][i] = clamp(n_vis[b][i] - shard_lo[b], 0, shard_len[b]).
 * n_vis int32 [B][Q]; shard_lo, shard_len int64 [B] (this rank's shard of each
 * sequence); n_vis_local int32 [B][Q].  A negative shard_lo or shard_len gives 0 and
 * flags CSA2_DEV_BAD_INDEX; a negative n_vis gives 0 and flags CSA2_DEV_BAD_COUNT. */
csa2_status csa2_cp_shard_vis(const int32_t* n_vis, const int64_t* shard_lo, const int64_t* shard_len, int B,
                              int Q, int32_t* n_vis_local, uint32_t* dev_status, cudaStream_t stream);

/* Merge of C candidate lists into the K best (P1 §무엇과 다른가, read as above).
 *   cand int32 [C][B][Q][Kc]: candidate labels local to shard c, -1 = empty slot
 *   cand_score fp32 [C][B][Q][Kc]: their scores
 *   part_stride  elements from shard c's list to shard c+1's, in both arrays (0 means
 *        B*Q*Kc, dense); a larger stride lets one gathered buffer per shard hold
 *        [labels | scores], so a single all-gather moves both
 *   shard_off int64 [C][B]: label offset of shard c in sequence b; the global label of
 *        a candidate is shard_off[c][b] + cand and must fit int32
 *   topk int32 [B][Q][K] out: global labels of the K best candidates (a set, -1 in
 *        unused slots); topk_score fp32 [B][Q][K] may be NULL
 * Order: larger score first (fp32 values compared exactly); equal scores prefer the
 * lower shard, then the earlier slot, which with lists from csa2_index_full or
 * csa2_index_hier over shards ordered by rank is the lower global label, as on one
 * device.  Candidates below -1 or whose label overflows are skipped and flag
 * CSA2_DEV_BAD_INDEX.  1 <= C <= CSA2_MAX_SHARDS, 1 <= Kc, K <= CSA2_MAX_K. */
size_t csa2_topk_merge_workspace_size(int C, int B, int Q, int Kc);
csa2_status csa2_topk_merge(const int32_t* cand, const float* cand_score, int64_t part_stride,
                            const int64_t* shard_off, int C, int B, int Q, int Kc, int K, int32_t* topk,
                            float* topk_score, void* ws, size_t ws_bytes, uint32_t* dev_status,
                            cudaStream_t stream);

/* This rank's part of a merged list: for every query, the labels t of topk int32
 * [B][Q][K] with shard_off[b] <= t < shard_off[b] + shard_len[b], as t - shard_off[b],
 * compacted to the front of topk_local int32 [B][Q][K] in slot order; -1 fills the
 * rest.  shard_off, shard_len int64 [B] (entry units; block units for block lists).
 * topk_local must not alias topk.  A negative offset or length gives an all-empty row
 * and flags CSA2_DEV_BAD_INDEX. */
csa2_status csa2_topk_localize(const int32_t* topk, int B, int Q, int K, const int64_t* shard_off,
                               const int64_t* shard_len, int32_t* topk_local, uint32_t* dev_status,
                               cudaStream_t stream);

/* Attention over the union of C disjoint key sets from each set's csa2_sparse_attn
 * result (P3 §전역 어텐션과 지역 어텐션: one softmax over all of a query's keys).
 *   out_parts fp32 [C][B][Q][H][512], lse_parts fp32 [C][B][Q][H] (natural log)
 *   out_part_stride  floats from part c to part c+1 of out_parts (0 means B*Q*H*512,
 *        dense; else at least that and a multiple of 4); lse_part_stride likewise for
 *        lse_parts (0 means B*Q*H): one gathered buffer per part can hold [out | lse]
 *   out fp32 [B][Q][H][512], lse fp32 [B][Q][H]; must not overlap the parts
 * With M = max_c lse_c: w_c = exp(lse_c - M), out = sum_c w_c out_c / sum_c w_c,
 * lse = M + log(sum_c w_c), in fp32.  Parts with lse_c = -inf add nothing; all parts
 * empty give out = 0, lse = -inf.  1 <= C <= CSA2_MAX_SHARDS. */
csa2_status csa2_attn_combine(const float* out_parts, int64_t out_part_stride, const float* lse_parts,
                              int64_t lse_part_stride, int C, int B, int Q, int H, float* out, float* lse,
                              cudaStream_t stream);

/* ---------------------------------------------------------------------------------
 * csa2_reindex_static: csa2_reindex without a workspace argument.  The pages have no
 * counterpart to this call; it is a library convenience for callers that cannot hand
 * the library device memory: a host with no device allocator of its own, or an engine
 * whose device memory is planned once before decoding and which must not ask for more
 * inside the decode loop.
 *
 * Arguments, layouts, results and device-side checks are those of csa2_reindex.  The
 * key scratch is a device array of CSA2_STATIC_SCRATCH_BYTES (4 MiB) compiled into the
 * library; every GPU on which the library's device code is loaded holds it until the
 * process exits.  Nothing is allocated by the call.
 *  - Size limit: when csa2_reindex_workspace_size(B, Q, HI, n_blocks, block, K) exceeds
 *    CSA2_STATIC_SCRATCH_BYTES the call returns CSA2_ERR_UNSUPPORTED before touching
 *    the device (n_blocks * block = 16,384 candidates fit 64 queries).
 *  - Set-up: the first call on a device, with that device current, looks up the array's
 *    device address (cudaGetSymbolAddress) and caches it for that device context;
 *    CSA2_ERR_CUDA if that fails.  A reset device (cudaDeviceReset) has a new context,
 *    so the first call after it looks the address up again.  Make the first call on
 *    each device, and the first after a reset, before any stream capture.
 *  - Nothing in the array needs to start at zero: the scan writes every key the
 *    selection reads back within the same call.
 *  - One array per device: calls whose kernels overlap on the same device (several
 *    streams or host threads) race on it and their results are undefined.  Issue the
 *    calls for one device on one stream.
 * csa2_static_scratch_bytes() returns CSA2_STATIC_SCRATCH_BYTES.
 * --------------------------------------------------------------------------------- */
size_t csa2_static_scratch_bytes(void);
csa2_status csa2_reindex_static(const float* q, const float* w, const uint8_t* ik_pool,
                                int64_t pool_entries, const int64_t* seq_base, const int32_t* n_vis,
                                const int32_t* blocks, int n_blocks, int block, int B, int Q, int HI,
                                int K, int32_t* topk, float* topk_score, uint32_t* dev_status,
                                cudaStream_t stream);

/* ---------------------------------------------------------------------------------
 * Test hook (no counterpart in the pages): csa2_index_full with one copy withheld.
 * The first CTA of the streaming scan never copies tile `withheld_tile` (>= 0) of its
 * run, so no barrier completes for it: the workers' bounded wait gives up (within about
 * a second), the scan drains what it issued, releases its tensor memory and sets
 * CSA2_DEV_TIMEOUT in *dev_status, and the selection that follows reads whatever keys
 * were written.  The call itself returns CSA2_OK once enqueued.  It exists so tests can
 * check that an expired device wait is reported and leaves the device usable; results
 * of the call are unspecified.  Arguments as for csa2_index_full.
 * --------------------------------------------------------------------------------- */
csa2_status csa2_test_index_full_withheld_copy(const float* q, const float* w, const uint8_t* ik_pool,
                                               int64_t pool_entries, const int64_t* seq_base,
                                               const int32_t* n_vis, int B, int Q, int HI, int K,
                                               int64_t max_n_vis, int32_t* topk, float* topk_score,
                                               void* ws, size_t ws_bytes, uint32_t* dev_status,
                                               cudaStream_t stream, int withheld_tile);

#ifdef __cplusplus
}
#endif

#endif /* CSA2_H */
