"""Plain CPU sampler of the denoising loop (the oracle's sampler half).

TEST INFRASTRUCTURE ONLY: only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA path.  Floating point is fp64; the random draws and every selection
are integer-exact.

Sources (the pages print no formula; each rule below is a reading of prose):

* Settings table "Configuracao de exibicao recomendada" on the Google docs
  page for DiffusionGemma: at most 48 denoising steps per canvas; temperature
  "Linear 0.8 -> 0.4" as a function of the step; adaptive stop when (A) the
  mean entropy over the canvas is below 0.005 and (B) two consecutive denoiser
  predictions are identical.
* aiexpert.news, "Google's DiffusionGemma Atinge 1.000 Tokens por Segundo",
  architecture paragraph: each forward pass locks in 15-20 high-confidence
  tokens, uses them as context for the rest, and may re-noise low-confidence
  positions in later passes.  The commit count here is k = 16 per pass and the
  re-noise threshold is a softmax confidence of 0.05.
* "DiffusionGemma Guia do Desenvolvedor ...", section "Demonstracao",
  bullet on re-noising: when confidence drops the sampler swaps the token for
  a random one.  Section "Difusao de Estado Uniforme": the canvas starts as
  random placeholders (uniform-state diffusion).

Readings (each listed in the design notes):
  T_s = t_start + (t_end - t_start) * s / (max_steps - 1), so step 0 runs at
      0.8 and step 47 at 0.4 exactly.
  z_v = l_v / T_s.  Entropy H = LSE(z) - sum_v p_v z_v in nats, p = softmax(z).
  Sample x_hat = argmax_v (z_v + g_v), g_v = -ln(-ln u_v) Gumbel noise from
      Philox (ties to the lowest index).
  Confidence (log form) lambda = z_x - LSE(z) with x = x_hat for positions
      uncommitted at the start of the step and x = the current token for
      committed ones.
  Commit the min(k, |U|) positions of the uncommitted set U with the largest
      lambda (ties to the lower position); they take x_hat.
  Re-noise R = {committed at step start with lambda < ln(0.05)}: a fresh
      uniform token, uncommitted again.
  Unselected uncommitted positions take x_hat and stay uncommitted (policy
      "keep"), or a fresh uniform token (policy "renoise").
  "Prediction" in stop rule (B) = the argmax of the raw logits at every position.
  Entropy-bounded selection (same settings table, row "Selecao de token":
      entropy limit 0.1, the lowest-entropy tokens are selected so that the
      mutual-information bound stays below the limit), used instead of the
      fixed k when selection = SELECT_ENTROPY: order U by entropy (ties to the
      lower position) and commit the longest prefix whose summed entropy is
      <= entropy_bound; at least the first position is committed, so that
      every step makes progress.
  Stop after step s when any of: every position is committed after the step;
      (A) and (B) with s >= 1; s = max_steps - 1.  On an (A)/(B) or step-cap
      stop every still-uncommitted position takes x_hat and is committed, and
      no re-noise happens in that step.
"""
from dataclasses import dataclass, field

import numpy as np

from .philox import (TAG_GUMBEL, TAG_INIT, TAG_RENOISE, position_word, token_from_word,
                     uniform_from_word, vocab_words)

POLICY_KEEP = 0
POLICY_RENOISE = 1

SELECT_TOP_K = 0     # the k uncommitted positions of largest confidence
SELECT_ENTROPY = 1   # lowest-entropy prefix within the entropy bound


@dataclass(frozen=True)
class SamplerCfg:
    max_steps: int = 48
    t_start: float = 0.8
    t_end: float = 0.4
    commit_k: int = 16
    renoise_conf: float = 0.05
    stop_entropy: float = 0.005
    unselected_policy: int = POLICY_KEEP
    selection: int = SELECT_TOP_K
    entropy_bound: float = 0.1


def temperature(cfg, step):
    """Linear schedule from t_start at step 0 to t_end at step max_steps - 1."""
    if cfg.max_steps <= 1:
        return cfg.t_start
    return cfg.t_start + (cfg.t_end - cfg.t_start) * step / (cfg.max_steps - 1)


def gumbel_noise(u):
    """g = -ln(-ln u); -ln u is taken through log1p above 1/2, where 1 - u is exact."""
    u = np.asarray(u, dtype=np.float64)
    e = np.where(u > 0.5, -np.log1p(-(1.0 - u)), -np.log(u))
    return -np.log(e)


def init_canvas(seed, b, block, canvas, vocab):
    """Uniform random placeholder tokens for a fresh canvas (Philox tag INIT)."""
    return np.array([token_from_word(position_word(seed, b, block, 0, i, TAG_INIT), vocab)
                     for i in range(canvas)], dtype=np.int64)


def renoise_token(seed, b, block, step, pos, vocab):
    return int(token_from_word(position_word(seed, b, block, step, pos, TAG_RENOISE), vocab))


@dataclass
class PositionStats:
    lse: float
    entropy: float
    argmax: int
    argmax_gap: float
    x_hat: int
    gumbel_gap: float
    z_xhat: float


def position_stats(row, temp, seed, b, block, step, pos):
    """Per-position statistics of one logits row (fp64 copy of the fp32 logits)."""
    row = np.asarray(row, dtype=np.float64)
    vocab = row.shape[0]
    z = row / temp
    m = np.max(z)
    lse = m + np.log(np.sum(np.exp(z - m)))
    p = np.exp(z - lse)
    entropy = lse - np.sum(p * z)
    a = int(np.argmax(row))
    if vocab > 1:
        second = np.max(np.delete(row, a))
        a_gap = float(row[a] - second)
    else:
        a_gap = np.inf
    u = uniform_from_word(vocab_words(seed, b, block, step, pos, TAG_GUMBEL, vocab))
    score = z + gumbel_noise(u)
    x = int(np.argmax(score))
    g_gap = float(score[x] - np.max(np.delete(score, x))) if vocab > 1 else np.inf
    return PositionStats(float(lse), float(entropy), a, a_gap, x, g_gap, float(z[x]))


@dataclass
class StepResult:
    tok: np.ndarray
    committed: np.ndarray
    argmax: np.ndarray
    x_hat: np.ndarray
    logconf: np.ndarray
    entropy: np.ndarray
    commit_mask: np.ndarray
    renoise_mask: np.ndarray
    stopped: bool
    reason: str
    near_tie: dict = field(default_factory=dict)


def sampler_step(cfg, logits, tok, committed, prev_argmax, step, seed, b, block, tie_margin=1e-4):
    """One sampler step of one sequence.

    logits [C, V] (fp32 values, any float dtype); tok [C] int; committed [C]
    bool; prev_argmax [C] int or None (no previous step).  Returns StepResult.
    """
    logits = np.asarray(logits, dtype=np.float64)
    C, V = logits.shape
    tok = np.asarray(tok, dtype=np.int64).copy()
    committed = np.asarray(committed, dtype=bool).copy()
    temp = temperature(cfg, step)

    stats = [position_stats(logits[i], temp, seed, b, block, step, i) for i in range(C)]
    lse = np.array([s.lse for s in stats])
    ent = np.array([s.entropy for s in stats])
    amax = np.array([s.argmax for s in stats], dtype=np.int64)
    xhat = np.array([s.x_hat for s in stats], dtype=np.int64)
    z_tok = logits[np.arange(C), tok] / temp
    z_x = np.array([s.z_xhat for s in stats])
    lam = np.where(committed, z_tok - lse, z_x - lse)

    uncommitted = np.flatnonzero(~committed)
    if cfg.selection == SELECT_ENTROPY:
        # Lowest entropy first, ties to the lower position; the longest prefix
        # whose entropies sum to at most the bound, and never an empty one.
        order = sorted(uncommitted.tolist(), key=lambda i: (ent[i], i))
        csum = np.cumsum([ent[i] for i in order])
        k = int(np.count_nonzero(csum <= cfg.entropy_bound))
        if uncommitted.size > 0:
            k = max(k, 1)
    else:
        k = min(cfg.commit_k, uncommitted.size)
        # Largest lambda first, ties to the lower position.
        order = sorted(uncommitted.tolist(), key=lambda i: (-lam[i], i))
    chosen = np.array(order[:k], dtype=np.int64)
    commit_mask = np.zeros(C, dtype=bool)
    commit_mask[chosen] = True

    mean_h = float(np.mean(ent))
    crit_a = mean_h < cfg.stop_entropy
    crit_b = prev_argmax is not None and step >= 1 and bool(np.all(amax == np.asarray(prev_argmax)))
    at_cap = step >= cfg.max_steps - 1

    log_tau = np.log(cfg.renoise_conf) if cfg.renoise_conf > 0 else -np.inf
    renoise_mask = np.zeros(C, dtype=bool)
    new_tok = tok.copy()
    new_comm = committed.copy()
    if (crit_a and crit_b) or at_cap:
        new_tok[~committed] = xhat[~committed]
        new_comm[:] = True
        stopped, reason = True, ("entropy" if (crit_a and crit_b) else "cap")
    else:
        new_tok[commit_mask] = xhat[commit_mask]
        new_comm[commit_mask] = True
        renoise_mask = committed & (lam < log_tau)
        for i in np.flatnonzero(renoise_mask):
            new_tok[i] = renoise_token(seed, b, block, step, i, V)
        new_comm[renoise_mask] = False
        unsel = (~committed) & (~commit_mask)
        if cfg.unselected_policy == POLICY_KEEP:
            new_tok[unsel] = xhat[unsel]
        else:
            for i in np.flatnonzero(unsel):
                new_tok[i] = renoise_token(seed, b, block, step, i, V)
        stopped = bool(np.all(new_comm))
        reason = "complete" if stopped else ""

    # Near-tie accounting: positions whose decision sits within tie_margin of
    # flipping (log space) are reported so a comparison can exclude them.
    near = {}
    near["gumbel"] = np.array([s.gumbel_gap < tie_margin for s in stats])
    near["argmax"] = np.array([s.argmax_gap < tie_margin for s in stats])
    boundary = np.zeros(C, dtype=bool)
    if cfg.selection == SELECT_ENTROPY:
        # the cut moves if an entropy sum straddles the bound, or if the last
        # selected and first unselected entropies nearly tie
        if 0 < k < uncommitted.size:
            e_in, e_out = ent[order[k - 1]], ent[order[k]]
            near_cut = (abs(csum[k] - cfg.entropy_bound) < tie_margin or
                        abs(csum[k - 1] - cfg.entropy_bound) < tie_margin or
                        (e_out - e_in) < tie_margin)
            if near_cut:
                boundary[np.array(order[k - 1:k + 1], dtype=np.int64)] = True
        elif 1 < k == uncommitted.size and abs(csum[k - 1] - cfg.entropy_bound) < tie_margin:
            # everything selected with the sum just under the bound: a slightly
            # larger sum would leave the last-ranked position out
            boundary[order[k - 1]] = True
    else:
        lam_u = np.sort(lam[uncommitted])[::-1]
        if 0 < k < uncommitted.size and (lam_u[k - 1] - lam_u[k]) < tie_margin:
            edge = 0.5 * (lam_u[k - 1] + lam_u[k])
            boundary[uncommitted[np.abs(lam[uncommitted] - edge) < tie_margin]] = True
    near["commit_boundary"] = boundary
    near["renoise"] = committed & (np.abs(lam - log_tau) < tie_margin)
    near["stop"] = abs(mean_h - cfg.stop_entropy) < tie_margin

    return StepResult(new_tok, new_comm, amax, xhat, lam, ent, commit_mask, renoise_mask,
                      stopped, reason, near)
