"""Temperature sampling for the draft-and-verify loop (fp64 CPU oracle).

TEST INFRASTRUCTURE ONLY: imported by tests/ (and, like the rest of this
package, never by the product package).

Sources.  [P2] iaemfoco.com, "DFlash: Decodificação Especulativa com Blocos em
Paralelo ...", section "Decodificação especulativa tradicional" (a small drafter
proposes future tokens, the target checks them in parallel, and the output is
the target's own) and section "Casos de uso" (the speed-up holds, smaller, when
sampling); [P4] imasters.com.br, "NVIDIA acelera LLMs autorregressivos em até
15 vezes", section "Os três mecanismos por trás do DFlash" (the target's output
distribution is kept).  The pages state no rule for sampling.  The reading here
is the standard speculative-sampling rule, the plainest one that keeps the
target's distribution exactly:

* temperature T > 0: P = softmax(target logits / T), Q = softmax(drafter logits / T);
* the drafter samples d_i ~ Q_i at block positions i = 1 .. B-1, all at once;
* for i = 1 .. B-1 in order, d_i is accepted with probability
  min(1, P_{i-1}(d_i) / Q_i(d_i)), where P_{i-1} is the target's distribution of
  verify row i-1 (the row whose next token is d_i);
* at the first rejection, at i, the token committed after d_1 .. d_{i-1} is
  drawn from max(0, P_{i-1} - Q_i), normalised; when all B-1 drafts are
  accepted, a bonus token is drawn from P_{B-1};
* the committed tokens are d_1 .. d_a and that one extra token (tau = a + 1),
  exactly as in greedy decoding, which this rule becomes as T -> 0.

Random numbers come from one counter-based generator, Philox4x32-10 (J. Salmon,
M. Moraes, R. Dror, D. Shaw, "Parallel random numbers: as easy as 1, 2, 3",
SC 2011), so that any implementation can draw the same numbers without passing
them around.  Key = the 64-bit seed (low word first).  Counter = (j, position,
sequence, purpose): word j % 4 of the block for counter word j // 4 gives draw
j of a vocabulary-wide vector; scalar draws use j = 0.  A 32-bit word w maps to
u = (floor(w / 512) + 1/2) * 2^-23 in [2^-24, 1 - 2^-24]: 23 random bits, each
value an odd 24-bit integer times 2^-24, so exact in fp32 as in fp64.
Draws use Gumbel-max: a sample from softmax(s) is argmax_v (s_v + G(u_v)) with
G(u) = -log(-log(u)), ties to the lowest index.  The position of a draw is the
absolute sequence position of the token it decides; purposes are below.  A
position's draws are used at most once for a committed decision: draws past the
first rejection of an iteration never influence a committed token, and the
positions up to it are committed.
"""
from typing import Callable, List, Optional, Tuple

import numpy as np

# purposes (counter word 3)
DRAFT = 1     # Gumbel noise of the drafter's sample at a position
ACCEPT = 2    # uniform deciding whether the draft at a position is accepted
RESIDUAL = 3  # Gumbel noise of the resample after a rejection at a position
TARGET = 4    # Gumbel noise of a token drawn from the target (first token, bonus, target-only decoding)

_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr, key) -> np.ndarray:
    """Philox4x32 with 10 rounds.  ctr: (..., 4) uint32, key: (..., 2) uint32
    (broadcast together); returns (..., 4) uint32.  Each round multiplies
    counter words 0 and 2 by the two Philox multipliers, swaps and XORs the
    high halves with the other words and the round key; the key is bumped by
    the two Weyl constants between rounds."""
    ctr = np.asarray(ctr, np.uint32)
    key = np.asarray(key, np.uint32)
    m0, m1 = np.uint64(0xD2511F53), np.uint64(0xCD9E8D57)
    w0, w1 = np.uint64(0x9E3779B9), np.uint64(0xBB67AE85)
    c0, c1, c2, c3 = (ctr[..., i].astype(np.uint64) for i in range(4))
    k0, k1 = key[..., 0].astype(np.uint64), key[..., 1].astype(np.uint64)
    for r in range(10):
        if r:
            k0 = (k0 + w0) & _MASK32
            k1 = (k1 + w1) & _MASK32
        p0 = m0 * c0  # exact: both factors < 2^32
        p1 = m1 * c2
        c0, c1, c2, c3 = ((p1 >> np.uint64(32)) ^ c1 ^ k0, p1 & _MASK32,
                          (p0 >> np.uint64(32)) ^ c3 ^ k1, p0 & _MASK32)
    c0, c1, c2, c3 = np.broadcast_arrays(c0, c1, c2, c3)
    return np.stack([c0, c1, c2, c3], -1).astype(np.uint32)


def word_to_uniform(w) -> np.ndarray:
    """u = (floor(w / 512) + 1/2) * 2^-23 in (0, 1): 23 random bits, exact in fp32."""
    w = np.asarray(w, np.uint32)
    return ((w >> np.uint32(9)).astype(np.float64) + 0.5) * 2.0 ** -23


def _key(seed: int) -> np.ndarray:
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return np.array([seed & 0xFFFFFFFF, seed >> 32], np.uint32)


def uniform_vector(seed: int, seq: int, pos: int, purpose: int, n: int) -> np.ndarray:
    """Draws j = 0 .. n-1 of (seed, seq, pos, purpose): uniforms in (0, 1)."""
    j = np.arange(n, dtype=np.uint64)
    ctr = np.zeros((len(range(0, n, 4)), 4), np.uint32)
    ctr[:, 0] = np.arange(ctr.shape[0], dtype=np.uint32)
    ctr[:, 1] = np.uint32(pos)
    ctr[:, 2] = np.uint32(seq)
    ctr[:, 3] = np.uint32(purpose)
    words = philox4x32_10(ctr, _key(seed))
    return word_to_uniform(words[(j >> np.uint64(2)).astype(np.int64), (j & np.uint64(3)).astype(np.int64)])


def uniform_scalar(seed: int, seq: int, pos: int, purpose: int) -> float:
    """Draw 0 of (seed, seq, pos, purpose)."""
    return float(uniform_vector(seed, seq, pos, purpose, 1)[0])


def gumbel(u) -> np.ndarray:
    """G(u) = -log(-log(u)): standard Gumbel variates from uniforms in (0, 1)."""
    return -np.log(-np.log(np.asarray(u, np.float64)))


def gumbel_argmax(scores, u) -> Tuple[int, float]:
    """argmax_v (scores_v + G(u_v)), lowest index on exact ties, and the margin
    between the two largest perturbed scores.  scores may hold -inf (excluded)."""
    y = np.asarray(scores, np.float64) + gumbel(u)
    i = int(np.argmax(y))  # numpy returns the first maximum
    if len(y) < 2:
        return i, float("inf")
    top2 = np.partition(y, -2)[-2:]
    return i, float(top2[1] - top2[0])


def softmax_t(logits, T: float) -> np.ndarray:
    """softmax(logits / T) in fp64 (rows along the last axis)."""
    z = np.asarray(logits, np.float64) / T
    z = z - z.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=-1, keepdims=True)


class Noise:
    """The draws of one sequence: seed (64-bit key) and sequence id (counter word 2)."""

    def __init__(self, seed: int, seq: int = 0):
        self.seed, self.seq = int(seed), int(seq)

    def vector(self, pos: int, purpose: int, n: int) -> np.ndarray:
        return uniform_vector(self.seed, self.seq, pos, purpose, n)

    def scalar(self, pos: int, purpose: int) -> float:
        return uniform_scalar(self.seed, self.seq, pos, purpose)


def sample_drafts(q_logits, T: float, p: int, noise: Noise) -> Tuple[np.ndarray, np.ndarray]:
    """Drafts d_1 .. d_{B-1} for an anchor at position p: d_i = argmax(z_i / T + G)
    with the DRAFT draws of position p + i.  Returns (drafts, Gumbel margins)."""
    q_logits = np.asarray(q_logits, np.float64)
    d = np.zeros(len(q_logits), np.int32)
    mg = np.zeros(len(q_logits))
    for i in range(1, len(q_logits) + 1):
        z = q_logits[i - 1]
        d[i - 1], mg[i - 1] = gumbel_argmax(z / T, noise.vector(p + i, DRAFT, len(z)))
    return d, mg


class BlockOutcome:
    """One iteration's decision: a accepted drafts, the extra token x, and how
    close each floating-point decision was (for comparisons across precisions)."""

    def __init__(self, a: int, x: int, accept_margins: List[float], x_margin: float, from_residual: bool):
        self.a, self.x = a, x
        self.accept_margins = accept_margins  # |u * Q(d) - P(d)| / Q(d) per decided draft
        self.x_margin = x_margin              # Gumbel margin of the extra token
        self.from_residual = from_residual

    @property
    def tau(self) -> int:
        return self.a + 1


def accept_block(P, Q, drafts, p: int, noise: Noise) -> BlockOutcome:
    """The speculative-sampling rule for an anchor at position p.
    P: [B, V] target probabilities of verify rows 0 .. B-1 (row i-1 is the
    distribution of the token at position p + i); Q: [B-1, V] drafter
    probabilities of positions p + 1 .. p + B - 1; drafts: d_1 .. d_{B-1}."""
    P = np.asarray(P, np.float64)
    Q = np.asarray(Q, np.float64)
    B = P.shape[0]
    margins = []
    for i in range(1, B):
        d = int(drafts[i - 1])
        pd, qd = P[i - 1, d], Q[i - 1, d]
        u = noise.scalar(p + i, ACCEPT)
        margins.append(abs(u * qd - pd) / qd if qd > 0 else float("inf"))
        if u * qd < pd:  # accepted with probability min(1, pd / qd)
            continue
        r = np.maximum(P[i - 1] - Q[i - 1], 0.0)
        pos_part = r > 0
        scores = np.full(r.shape, -np.inf)
        scores[pos_part] = np.log(r[pos_part])
        x, xm = gumbel_argmax(scores, noise.vector(p + i, RESIDUAL, len(r)))
        return BlockOutcome(i - 1, x, margins, xm, True)
    with np.errstate(divide="ignore"):
        scores = np.log(P[B - 1])
    x, xm = gumbel_argmax(scores, noise.vector(p + B, TARGET, P.shape[1]))
    return BlockOutcome(B - 1, x, margins, xm, False)


def sample_target(logits, T: float, pos: int, noise: Noise) -> Tuple[int, float]:
    """A token from softmax(logits / T) with the TARGET draws of its position."""
    z = np.asarray(logits, np.float64)
    return gumbel_argmax(z / T, noise.vector(pos, TARGET, len(z)))


# ---------------------------------------------------------------- whole generations
def generate_ar_sample(spec, prompt, max_new: int, T: float, seed: int, seq: int = 0):
    """Target-only sampling: token at position t from softmax(logits / T) with
    the TARGET draws of position t.  Uses the oracle's verify on one live row
    (row 0 of a block is causal in the tokens before it).  Returns (tokens, margins)."""
    cfg = spec.cfg
    noise = Noise(seed, seq)
    n = len(prompt)
    ss = spec.session(n + max_new + cfg.block_size + 1)
    _, _, lg = ss.prefill(prompt, want_logits=True)
    out, mg = [], []
    t, m = sample_target(lg, T, n, noise)
    out.append(t), mg.append(m)
    while len(out) < max_new:
        pos = ss.len
        block = [out[-1]] + [cfg.mask_id] * (cfg.block_size - 1)
        _, _, rows = ss.verify(block, want_logits=True)
        ss.commit(0)
        t, m = sample_target(rows[0], T, pos + 1, noise)
        out.append(t), mg.append(m)
    return np.array(out, np.int32), np.array(mg)


def generate_spec_sample(spec, prompt, max_new: int, T: float, seed: int, seq: int = 0,
                         log: Optional[Callable] = None):
    """Draft-and-verify sampling with the oracle's drafter and target.  Each
    iteration: drafter logits -> drafts (DRAFT draws), target verify of
    [anchor, drafts] -> the acceptance rule -> commit a + 1 rows.  log, when
    given, receives (p, drafts, draft_margins, outcome) per iteration.
    Returns (tokens, accept lengths a per iteration)."""
    cfg = spec.cfg
    noise = Noise(seed, seq)
    n = len(prompt)
    ss = spec.session(n + max_new + 2 * cfg.block_size)
    _, _, lg = ss.prefill(prompt, want_logits=True)
    anchor, _ = sample_target(lg, T, n, noise)
    out, acc = [anchor], []
    while len(out) < max_new:
        p = ss.len
        _, _, q_logits = ss.draft(anchor, want_logits=True)
        drafts, dmg = sample_drafts(q_logits, T, p, noise)
        _, _, p_logits = ss.verify([anchor] + [int(d) for d in drafts], want_logits=True)
        o = accept_block(softmax_t(p_logits, T), softmax_t(q_logits, T), drafts, p, noise)
        if log:
            log(p, drafts, dmg, o)
        ss.commit(o.a)
        out.extend(int(d) for d in drafts[:o.a])
        out.append(o.x)
        acc.append(o.a)
        anchor = o.x
    return np.array(out[:max_new], np.int32), np.array(acc, np.int32)
