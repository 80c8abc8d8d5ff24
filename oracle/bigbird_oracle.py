"""fp64 CPU oracle for BigBird ITC block-sparse attention, forward and backward.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only the tests, the smoke check and the CPU-baseline leg
of the benchmark do.  It shares no code with the CUDA library.

What it computes, and where the pages state it
----------------------------------------------
Sources (web pages; titles and sections):

* [GC] "models 仓库中的 BigBird：线性复杂度稀疏注意力与长序列训练的完整实践"
  (blog.gitcode.com), section "BigBird：从二次方注意力到线性稀疏注意力":
  the three-part pattern (banded window of 3 blocks around the query block,
  first and last blocks global, num_rand_blocks random blocks that are not
  adjacent), the five segments first / second / middle / second_last / last,
  and masked positions receiving a -10000 offset before the softmax.
* [GC] section "随机块掩码是如何生成的": random blocks are drawn per head from
  the block ids without the first and last block, excluding the row's own
  window; the blocked key mask is the [B, L] mask reshaped to
  [B, L/bs, bs].
* [XZ] "Big Bird: Transformers for Longer Sequences" paper card
  (ai-papers.xuzou.cn), section "方法适配": queries/keys are blockified and the
  attended block budget per query block is constant, so work is linear in L.

Readings taken where the pages are silent:

* The attended set A(i) of query block i is a SET of key blocks: rows 0 and
  nb-1 (global) attend every block; every other row attends
  {i-1, i, i+1} U {0, nb-1} U rand[h, i, :r_eff], each block once.  The
  "second" and "second_last" segments exist because the window of rows 1
  and nb-2 overlaps a global block; union means no double counting.
* score s_tu = scale * <q_t, k_u> + (key_mask[b, u] ? 0 : mask_value),
  scale = 1/sqrt(d) by default, mask_value = -10000 by default.  The scale is
  applied before the offset; the offset is not scaled.  Blocks outside A(i)
  are absent (as if -inf), masked keys inside A(i) get the finite offset.
* lse_t = ln sum_u exp(s_tu) over the attended keys (natural log).
* The key mask is key-side only by default: query rows of padding are
  computed like any other row.  The optional query_mask (the from-side mask
  BigBirdMasks derives from the same input mask, [GC]
  随机块掩码是如何生成的) zeroes the output rows of padding tokens, so they
  pass no gradient.
* The random table follows this library's own specification (the pages'
  NumPy stream is not given): per head h and middle row i, the candidates are
  the ascending block ids j in [1, nb-2] with |j - i| > 1; a SplitMix64
  stream (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014) is seeded with seed XOR ((h << 32) | i); a partial
  Fisher-Yates shuffle draws r_eff = min(r, |cand|) of them; the chosen ids
  are written sorted ascending, unused slots and rows 0 and nb-1 hold -1.

* The pages' layer draws its table once for the maximum length
  (max_rand_mask_length = max_position_embeddings), with random blocks
  restricted to tokens before last_idx = 1024, and uses its first rows for
  a shorter sequence ([GC] 随机块掩码是如何生成的).  Both are options of
  rand_table (off by default): rows drawn for max_blocks blocks with ids
  below last_block; a row keeps the drawn ids that are middle blocks of the
  shorter table (an id at its last block is global already, one past it
  does not exist).
* Attention dropout ([GC] sections "BigBirdEncoder 的关键参数", which lists
  attention_dropout_rate = 0.1, and "梯度检查点的实现方式", which requires
  stateless, seeded dropout so a recomputed forward draws the same noise):
  the dropout multiplies the attended softmax probabilities by 0 (dropped)
  or 1 / keep probability (kept); the lse is that of the undropped softmax.
  The keep decision of element (b, h, t, u) is this library's own
  specification (the pages give no generator): Philox4x32-10 (Salmon et
  al., SC 2011) with counter (u >> 4, t, h, b) and the 64-bit seed as key;
  byte u & 15 of its 16 little-endian output bytes is compared with the
  rate rounded to 1/256 (dropped when below).

The backward pass is the gradient of the forward's definition (the pages do
not spell it out; the pages' layer trains with autodiff and recomputation):
D_t = <dO_t, o_t>, dS_tu = p_tu (<dO_t, v_u> - D_t), dq_t = scale sum_u
dS_tu k_u, dk_u = scale sum_t dS_tu q_t, dv_u = sum_t p_tu dO_t.

Pins: tests/test_oracle.py checks this module against brute-force dense
masked softmax attention, torch fp64 autograd, finite differences, library
SDPA on the shapes where the pattern is dense, a closed-form adjacency
read-out and invariants; tests/test_rand_table.py checks the generator
against the published SplitMix64 outputs and the table's defining
properties; tests/test_dropout_oracle.py checks the dropout generator
against the published Philox4x32-10 known-answer vectors and the dropped
forward and backward against dense torch fp64 with autograd and finite
differences; tests/test_query_mask_oracle.py does the same for the query
mask; tests/test_proj_oracle.py checks the projections against explicit
element-by-element sums and identity-weight read-outs.
"""

import math

import numpy as np

_MASK64 = (1 << 64) - 1
# SplitMix64 constants from the published generator (Steele, Lea and Flood
# 2014; the public-domain reference code by S. Vigna): golden-ratio
# increment and the two multipliers of the output mix.
_SM64_GAMMA = 0x9E3779B97F4A7C15
_SM64_MUL1 = 0xBF58476D1CE4E5B9
_SM64_MUL2 = 0x94D049BB133111EB

DEFAULT_MASK_VALUE = -10000.0


class SplitMix64:
    """SplitMix64 stream: advance the state by the golden gamma, then mix."""

    def __init__(self, state):
        self.state = int(state) & _MASK64

    def next(self):
        self.state = (self.state + _SM64_GAMMA) & _MASK64
        z = self.state
        z = ((z ^ (z >> 30)) * _SM64_MUL1) & _MASK64
        z = ((z ^ (z >> 27)) * _SM64_MUL2) & _MASK64
        return z ^ (z >> 31)


def random_candidates(i, num_blocks):
    """Block ids a middle row i may draw at random ([GC] 随机块掩码是如何生成的):
    the middle blocks [1, nb-2] (first and last dropped) minus the row's own
    window {i-1, i, i+1}, ascending."""
    return [j for j in range(1, num_blocks - 1) if abs(j - i) > 1]


def rand_table(seed, heads, num_blocks, r, max_blocks=0, last_block=0):
    """int32 [heads, num_blocks, r] random block table (spec in module doc).

    max_blocks, last_block (0 = off): the options of the pages' layer ([GC]
    随机块掩码是如何生成的: the table is drawn once for the maximum length,
    with random blocks before token last_idx, and its first rows are used
    for a shorter sequence).  Row i is drawn as in a table of max_blocks
    blocks whose candidates are also below last_block; it keeps the drawn
    ids that are middle blocks of this table (<= num_blocks - 2), sorted."""
    if heads < 0 or num_blocks < 0 or r < 0 or max_blocks < 0 or last_block < 0:
        raise ValueError("negative size")
    nbb = max_blocks or num_blocks
    if nbb < num_blocks:
        raise ValueError("max_blocks below num_blocks")
    table = np.full((heads, num_blocks, r), -1, dtype=np.int32)
    for h in range(heads):
        for i in range(1, num_blocks - 1):
            cand = random_candidates(i, nbb)
            if last_block:
                cand = [j for j in cand if j < last_block]
            r_eff = min(r, len(cand))
            rng = SplitMix64((int(seed) ^ ((h << 32) | i)) & _MASK64)
            for kk in range(r_eff):
                u = rng.next()
                t = kk + u % (len(cand) - kk)
                cand[kk], cand[t] = cand[t], cand[kk]
            kept = sorted(j for j in cand[:r_eff] if j <= num_blocks - 2)
            table[h, i, :len(kept)] = kept
    return table


def attended_blocks(i, num_blocks, rand_row):
    """Sorted set A(i) of key blocks query block i attends ([GC] 从二次方注意力
    到线性稀疏注意力; union reading for rows 1 and nb-2)."""
    if i == 0 or i == num_blocks - 1:
        return list(range(num_blocks))
    s = {i - 1, i, i + 1, 0, num_blocks - 1}
    s.update(int(j) for j in rand_row if j >= 0)
    return sorted(j for j in s if 0 <= j < num_blocks)


# ---------------------------------------------------------------------------
# Seeded attention dropout.
#
# [GC] section "BigBirdEncoder 的关键参数" lists attention_dropout_rate (0.1 by
# default) beside the ordinary dropout rate; section "梯度检查点的实现方式"
# explains that, under recomputation, the dropout must be stateless and
# seeded so that the recomputed forward draws the same noise.  Readings
# taken: the dropout acts on the softmax probabilities of the
# attended keys (the usual attention dropout), the lse stays that of the
# undropped softmax, and the keep decision of element (b, h, t, u) is a pure
# function of (seed, b, h, t, u), drawn from Philox4x32-10 as specified below.
# ---------------------------------------------------------------------------

_MASK32 = 0xFFFFFFFF
# Philox4x32 constants from the published generator (J. K. Salmon,
# M. A. Moraes, R. O. Dror and D. E. Shaw, "Parallel random numbers: as easy
# as 1, 2, 3", SC 2011): the two round multipliers and the two Weyl
# increments of the key schedule.
_PHILOX_M0 = 0xD2511F53
_PHILOX_M1 = 0xCD9E8D57
_PHILOX_W0 = 0x9E3779B9
_PHILOX_W1 = 0xBB67AE85


def philox4x32_10(ctr, key):
    """Philox4x32 with 10 rounds on arrays of counters.

    ctr: four arrays (broadcastable, values < 2**32) c0..c3; key: two ints
    k0, k1.  Returns the four output words as uint64 arrays holding 32-bit
    values.  Each round multiplies c0 by M0 and c2 by M1 into 64-bit
    products; the new words are (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2),
    hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)); between rounds the key advances by the
    Weyl increments (W0, W1) modulo 2**32."""
    c = [np.asarray(x, dtype=np.uint64) & np.uint64(_MASK32) for x in ctr]
    c = list(np.broadcast_arrays(*c))
    k0 = int(key[0]) & _MASK32
    k1 = int(key[1]) & _MASK32
    m32 = np.uint64(_MASK32)
    sh = np.uint64(32)
    for rnd in range(10):
        if rnd:
            k0 = (k0 + _PHILOX_W0) & _MASK32
            k1 = (k1 + _PHILOX_W1) & _MASK32
        p0 = c[0] * np.uint64(_PHILOX_M0)  # < 2**64: exact in uint64
        p1 = c[2] * np.uint64(_PHILOX_M1)
        c = [(p1 >> sh) ^ c[1] ^ np.uint64(k0), p1 & m32,
             (p0 >> sh) ^ c[3] ^ np.uint64(k1), p0 & m32]
    return c


def dropout_threshold(rate):
    """Byte threshold of a dropout rate: the rate rounded to the nearest
    multiple of 1/256 (halves up), as an integer thr in [0, 255]; an element
    is dropped when its byte is below thr."""
    rate = float(rate)
    if not 0.0 <= rate < 1.0:
        raise ValueError("dropout rate must be in [0, 1)")
    thr = int(math.floor(rate * 256.0 + 0.5))
    if thr > 255:
        raise ValueError("dropout rate rounds to 1")
    return thr


def dropout_scale(rate):
    """Factor applied to kept probabilities: 1 / keep probability, with the
    keep probability (256 - thr) / 256 of the rounded rate, so the dropped
    probabilities are unbiased."""
    return 256.0 / (256 - dropout_threshold(rate))


def dropout_keep(seed, b, h, rows, cols, rate):
    """bool [len(rows), len(cols)] keep decisions of query tokens rows and key
    tokens cols of batch b, head h.

    Element (b, h, t, u) draws Philox4x32-10 with counter
    (u >> 4, t, h, b) and key (seed mod 2**32, seed >> 32); the 16 output
    bytes, taken little-endian from the words in order, belong to the key
    tokens 16 (u >> 4) .. 16 (u >> 4) + 15, and byte u & 15 decides.  The
    element is kept when its byte is >= dropout_threshold(rate)."""
    thr = dropout_threshold(rate)
    seed = int(seed) & _MASK64
    t = np.asarray(rows, dtype=np.uint64)[:, None]
    u = np.asarray(cols, dtype=np.uint64)[None, :]
    words = philox4x32_10((u >> np.uint64(4), t, np.uint64(h), np.uint64(b)),
                          (seed & _MASK32, seed >> 32))
    j = (u & np.uint64(15)).astype(np.int64)
    w = np.choose(np.broadcast_to(j >> 2, words[0].shape), words)
    byte = (w >> (np.uint64(8) * (u & np.uint64(3)))) & np.uint64(0xFF)
    return byte >= np.uint64(thr)


class Dropout:
    """Attention dropout of one call: rate in [0, 1) and a 64-bit seed.

    b0, h0: index offsets for a (b, h) slice computed as a problem of its
    own, so that its decisions are those of batch b0 + b, head h0 + h of the
    whole call."""

    def __init__(self, rate, seed, b0=0, h0=0):
        dropout_threshold(rate)  # validates
        self.rate = float(rate)
        self.seed = int(seed) & _MASK64
        self.b0, self.h0 = int(b0), int(h0)

    def factors(self, b, h, rows, cols):
        """[len(rows), len(cols)] multipliers of the probabilities: the
        scale where kept, 0 where dropped."""
        keep = dropout_keep(self.seed, self.b0 + b, self.h0 + h, rows, cols,
                            self.rate)
        return np.where(keep, dropout_scale(self.rate), 0.0)


def _prep(x):
    return np.asarray(x, dtype=np.float64)


def _key_offsets(key_mask, B, L, mask_value):
    """Additive offset per key: 0 where attended, mask_value where masked."""
    if key_mask is None:
        return np.zeros((B, L), dtype=np.float64)
    km = np.asarray(key_mask).reshape(B, L).astype(bool)
    return np.where(km, 0.0, float(mask_value))


def _token_cols(blocks, bs):
    return np.concatenate([np.arange(j * bs, (j + 1) * bs) for j in blocks])


def block_probs(q, k, key_mask, table, block_size, b, h, i, scale=None,
                mask_value=DEFAULT_MASK_VALUE):
    """Softmax probabilities of query block i of (b, h).

    Returns (key token indices, p [bs, n_keys], lse [bs]).  Softmax is taken
    in fp64 with the row maximum subtracted."""
    q = _prep(q)
    k = _prep(k)
    B, H, L, d = q.shape
    bs = block_size
    nb = L // bs
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    off = _key_offsets(key_mask, B, L, mask_value)
    cols = _token_cols(attended_blocks(i, nb, table[h, i]), bs)
    qi = q[b, h, i * bs:(i + 1) * bs]
    s = scale * (qi @ k[b, h, cols].T) + off[b, cols][None, :]
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    return cols, e / z, (m + np.log(z))[:, 0]


def _query_factors(query_mask, B, L):
    """[B, L] 1.0 for real query tokens, 0.0 for padding (None: all real)."""
    if query_mask is None:
        return np.ones((B, L))
    return (np.asarray(query_mask).reshape(B, L) != 0).astype(np.float64)


def forward(q, k, v, key_mask, table, block_size, scale=None,
            mask_value=DEFAULT_MASK_VALUE, dropout=None, query_mask=None):
    """Block-sparse attention forward: (o [B,H,L,d], lse [B,H,L]) in fp64.

    q, k, v: [B, H, L, d] (any float dtype, read as fp64); key_mask: None or
    [B, L] with nonzero = attend; table: int [H, nb, r].  dropout: None or a
    Dropout; o then sums the kept probabilities times the dropout scale,
    while lse stays that of the undropped softmax.  query_mask: None or
    [B, L], nonzero = real token: rows of padding tokens output zero (the
    from-side mask of [GC] 随机块掩码是如何生成的, where BigBirdMasks derives
    the from and to masks of the attention from the same input mask); their
    lse is still the row's normaliser."""
    q = _prep(q)
    k = _prep(k)
    v = _prep(v)
    B, H, L, d = q.shape
    bs = block_size
    if L % bs:
        raise ValueError("L must be a multiple of block_size")
    nb = L // bs
    qf = _query_factors(query_mask, B, L)
    o = np.zeros((B, H, L, d))
    lse = np.zeros((B, H, L))
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                cols, p, l = block_probs(q, k, key_mask, table, bs, b, h, i,
                                         scale, mask_value)
                if dropout is not None:
                    p = p * dropout.factors(b, h, np.arange(i * bs, (i + 1) * bs),
                                            cols)
                rows = slice(i * bs, (i + 1) * bs)
                o[b, h, rows] = qf[b, rows][:, None] * (p @ v[b, h, cols])
                lse[b, h, rows] = l
    return o, lse


def backward(q, k, v, dout, key_mask, table, block_size, scale=None,
             mask_value=DEFAULT_MASK_VALUE, dropout=None, query_mask=None):
    """Gradient of forward's o with respect to q, k, v for upstream dout.

    Returns (dq, dk, dv), each [B, H, L, d] fp64.  Probabilities and o are
    recomputed here from the definition, in fp64.  With dropout (factors
    m_tu: the scale where kept, 0 where dropped) o_t = sum_u m_tu p_tu v_u,
    so D_t = <dO_t, o_t> still, dS_tu = p_tu (m_tu <dO_t, v_u> - D_t) and
    dv_u = sum_t m_tu p_tu dO_t.  With query_mask the output row of a
    padding token is multiplied by 0, so its dO_t enters as 0: its dq is 0
    and it adds nothing to dk, dv."""
    q = _prep(q)
    k = _prep(k)
    v = _prep(v)
    dout = _prep(dout)
    B, H, L, d = q.shape
    bs = block_size
    nb = L // bs
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    qf = _query_factors(query_mask, B, L)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                cols, p, _ = block_probs(q, k, key_mask, table, bs, b, h, i,
                                         scale, mask_value)
                rows = slice(i * bs, (i + 1) * bs)
                vc = v[b, h, cols]
                kc = k[b, h, cols]
                do_i = qf[b, rows][:, None] * dout[b, h, rows]
                m = 1.0
                if dropout is not None:
                    m = dropout.factors(b, h, np.arange(i * bs, (i + 1) * bs),
                                        cols)
                o_i = (m * p) @ vc
                D = (do_i * o_i).sum(axis=1)
                dP = m * (do_i @ vc.T)
                dS = p * (dP - D[:, None])
                dq[b, h, rows] = scale * (dS @ kc)
                # cols holds each key token once, so fancy-index += is exact.
                dk[b, h, cols] += scale * (dS.T @ q[b, h, rows])
                dv[b, h, cols] += (m * p).T @ do_i
    return dq, dk, dv


def pair_count(num_blocks, table_h):
    """Number of attended (query block, key block) pairs for one head."""
    return sum(len(attended_blocks(i, num_blocks, table_h[i]))
               for i in range(num_blocks))


# ---------------------------------------------------------------------------
# The projections on either side of the attention.
#
# [GC] section "两条构建路径：EncoderScaffold 与 BigBirdEncoder": the encoder
# layer is a transformer block whose attention is BigBirdAttention, with
# key_dim = hidden / num_heads; its query, key and value are dense layers of
# the layer input, split into heads, and its output is a dense layer of the
# concatenated heads.  Written here as plain fp64 matrix products with the
# linear-layer weight convention W[out_features][in_features].
# ---------------------------------------------------------------------------


def qkv_projection(x, w_qkv, b_qkv, heads, head_dim=64):
    """q, k, v [B, H, L, head_dim] of x [B, L, hidden].

    w_qkv [3 * H * head_dim, hidden]: rows 0 .. D-1 produce the query
    features (D = H * head_dim; feature h * head_dim + j is component j of
    head h), rows D .. 2D-1 the key features, rows 2D .. 3D-1 the value
    features; b_qkv [3D] or None."""
    x = _prep(x)
    w = _prep(w_qkv)
    B, L, _ = x.shape
    D = heads * head_dim
    y = x @ w.T
    if b_qkv is not None:
        y = y + _prep(b_qkv)
    out = []
    for part in range(3):
        z = y[:, :, part * D:(part + 1) * D].reshape(B, L, heads, head_dim)
        out.append(np.ascontiguousarray(z.transpose(0, 2, 1, 3)))
    return tuple(out)


def output_projection(o, w_o, b_o):
    """out [B, L, hidden] of the attention output o [B, H, L, head_dim]:
    the heads concatenated per token (feature h * head_dim + j), times
    w_o [hidden, H * head_dim] transposed, plus b_o [hidden] or None."""
    o = _prep(o)
    B, H, L, d = o.shape
    cat = o.transpose(0, 2, 1, 3).reshape(B, L, H * d)
    y = cat @ _prep(w_o).T
    if b_o is not None:
        y = y + _prep(b_o)
    return y
