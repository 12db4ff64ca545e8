"""Learning the reference queries against a teacher: the CPU oracle.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT. Like the rest of ``oracle/``, only
``tests/``, the smoke check and ``bench.py``'s CPU legs may import it; it shares no
code with the CUDA library.

Page "How does a tree of summaries search a context? How ZHA works", section
"Does the model have to be retrained?": the model stays frozen and only the
reference queries are learned, by comparing how the tree splits attention with how
the model does (KL distillation). The pages give no more than that. The reading
taken here, written out plainly in double precision with torch's autograd for the
gradient:

- the tree is built from the keys and the reference queries exactly as in the
  build (page section "What does a node summarize?"): for each node and reference
  q_r, child scores s_i = beta*<key_i, q_r> + bias_i (bias 0 for keys),
  w = softmax(s), key_r = sum_i w_i key_i, bias_r = logsumexp(s) - beta*<key_r, q_r>;
- at every level l, for a query q, the tree splits attention over the level's
  nodes as softmax_j(score_j), score_j = max_r(beta*<key_{j,r}, q> + bias_{j,r})
  (section "What does a node summarize?");
- the teacher (the frozen model) splits it as the dense attention mass under each
  node: P_j = sum over the keys under node j of softmax_i(beta*<q, k_i>), the
  softmax taken over the keys the level covers (C^l * n_l of them);
- the loss is KL(P || tree split) summed over the levels and averaged over the
  queries; gradient steps on the reference queries lower it.
"""
from __future__ import annotations

import torch


def build_levels(K: torch.Tensor, refs: torch.Tensor, C: int, depth: int, beta: float):
    """Node keys [n_l][R][d] and biases [n_l][R] of levels 1..depth, built from the
    keys K [N][d] and references refs [R][d] (double precision, differentiable)."""
    R, d = refs.shape
    levels = []
    child_k = K[None].expand(R, -1, -1)  # [R][n][d]: leaves are shared by every reference
    child_b = torch.zeros(R, K.shape[0], dtype=K.dtype)
    for _ in range(depth):
        n = child_k.shape[1] // C
        if n == 0:
            levels.append((torch.zeros(0, R, d, dtype=K.dtype), torch.zeros(0, R, dtype=K.dtype)))
            child_k = child_k[:, :0]
            child_b = child_b[:, :0]
            continue
        ck = child_k[:, : n * C].reshape(R, n, C, d)
        cb = child_b[:, : n * C].reshape(R, n, C)
        s = beta * torch.einsum("rncd,rd->rnc", ck, refs) + cb
        w = torch.softmax(s, dim=2)
        key = torch.einsum("rnc,rncd->rnd", w, ck)
        bias = torch.logsumexp(s, dim=2) - beta * torch.einsum("rnd,rd->rn", key, refs)
        levels.append((key.permute(1, 0, 2), bias.t()))
        child_k, child_b = key, bias
    return levels


def split_loss(K: torch.Tensor, refs: torch.Tensor, Q: torch.Tensor, C: int, depth: int, beta: float,
               per_level: bool = False):
    """Mean over the queries Q [m][d] of sum over levels of KL(teacher split || tree
    split); with per_level, the [depth] vector of level terms instead of the sum."""
    levels = build_levels(K, refs, C, depth, beta)
    logits = beta * Q @ K.t()  # [m][N] dense attention scores
    terms = []
    for l, (key, bias) in enumerate(levels, start=1):
        n = key.shape[0]
        if n == 0:
            terms.append(torch.zeros((), dtype=K.dtype))
            continue
        span = C ** l
        covered = logits[:, : n * span]
        # teacher: dense mass under each node, over the keys the level covers
        logP = torch.logsumexp(covered.reshape(-1, n, span), dim=2)
        logP = logP - torch.logsumexp(logP, dim=1, keepdim=True)
        # tree: softmax over the level's node scores
        score = (beta * torch.einsum("jrd,md->mjr", key, Q) + bias[None]).amax(dim=2)
        logT = torch.log_softmax(score, dim=1)
        terms.append((logP.exp() * (logP - logT)).sum(dim=1).mean())
    terms = torch.stack(terms)
    return terms if per_level else terms.sum()


def learn_refs(K: torch.Tensor, refs0: torch.Tensor, Q: torch.Tensor, C: int, depth: int, beta: float,
               steps: int, lr: float):
    """Plain gradient descent on the reference queries; returns (refs, losses)."""
    refs = refs0.clone().requires_grad_(True)
    losses = []
    for _ in range(steps):
        loss = split_loss(K, refs, Q, C, depth, beta)
        (g,) = torch.autograd.grad(loss, refs)
        losses.append(float(loss.detach()))
        with torch.no_grad():
            refs -= lr * g
    losses.append(float(split_loss(K, refs.detach(), Q, C, depth, beta)))
    return refs.detach(), losses


def _lse(x, axis: int):
    import numpy as np

    m = x.max(axis=axis, keepdims=True)
    return np.log(np.exp(x - m).sum(axis=axis)) + np.squeeze(m, axis=axis)


def split_loss_and_grad(K, refs, Q, C: int, depth: int, beta: float):
    """The split loss and its gradient with respect to the references, written out
    (numpy, double precision, no autograd): the backward pass a GPU version
    follows. Per level l and query m, with g = (tree split - teacher split) / m_q
    on the node scores:
      - a node score is beta*<key_{j,r*}, q> + bias_{j,r*} at its best reference
        r*, so g flows to key_{j,r*} as g*beta*q and to bias_{j,r*} as g;
      - a node (j, r) built from children i with s_i = beta*<c_i, q_r> + b_i,
        w = softmax(s), key = sum_i w_i c_i, bias = logsumexp(s) - beta*<key, q_r>
        passes on, with Gk = G_key - beta*G_bias*q_r and
        G_s_i = w_i*(<Gk, c_i> - <Gk, key> + G_bias):
          to its children: G_c_i += w_i*Gk + beta*G_s_i*q_r, G_b_i += G_s_i;
          to its reference: G_q_r += beta*(sum_i G_s_i*c_i - G_bias*key);
    taken from the top level down, each level's node gradients being its own loss
    term's plus what its parents pass on. Returns (loss, gradient [R][d])."""
    import numpy as np

    K = np.asarray(K, dtype=np.float64)
    refs = np.asarray(refs, dtype=np.float64)
    Q = np.asarray(Q, dtype=np.float64)
    R, d = refs.shape
    m_q = Q.shape[0]
    # forward, keeping every level's children
    levels = []  # (child keys [R][n][C][d], child biases [R][n][C], w [R][n][C], key [R][n][d])
    ck_all = np.broadcast_to(K[None], (R,) + K.shape)
    cb_all = np.zeros((R, K.shape[0]))
    for _ in range(depth):
        n = ck_all.shape[1] // C
        ck = ck_all[:, : n * C].reshape(R, n, C, d)
        cb = cb_all[:, : n * C].reshape(R, n, C)
        s = beta * np.einsum("rncd,rd->rnc", ck, refs) + cb
        lse = _lse(s, 2) if n else np.zeros((R, 0))
        w = np.exp(s - lse[..., None])
        key = np.einsum("rnc,rncd->rnd", w, ck)
        bias = lse - beta * np.einsum("rnd,rd->rn", key, refs)
        levels.append((ck, cb, w, key, bias))
        ck_all, cb_all = key, bias
    # loss terms and the score gradients of every level
    logits = beta * Q @ K.T
    loss = 0.0
    G_key = [np.zeros_like(lv[3]) for lv in levels]   # [R][n][d] per level
    G_bias = [np.zeros_like(lv[4]) for lv in levels]  # [R][n]
    for li, (ck, cb, w, key, bias) in enumerate(levels):
        n = key.shape[1]
        if n == 0:
            continue
        span = C ** (li + 1)
        blocks = logits[:, : n * span].reshape(m_q, n, span)
        logP = _lse(blocks, 2)                    # log dense mass under each node
        logP = logP - _lse(logP, 1)[:, None]      # over the keys the level covers
        per_r = beta * np.einsum("rnd,md->mnr", key, Q) + bias.T[None]  # [m][n][R]
        best = per_r.argmax(axis=2)
        score = np.take_along_axis(per_r, best[..., None], axis=2)[..., 0]
        logT = score - _lse(score, 1)[:, None]
        P = np.exp(logP)
        loss += float((P * (logP - logT)).sum(axis=1).mean())
        g = (np.exp(logT) - P) / m_q  # [m][n]
        for r in range(R):
            sel = (best == r) * g  # [m][n]
            G_key[li][r] += beta * sel.T @ Q
            G_bias[li][r] += sel.sum(axis=0)
    # backward through the build, top level first
    grad = np.zeros_like(refs)
    for li in range(len(levels) - 1, -1, -1):
        ck, cb, w, key, bias = levels[li]
        if key.shape[1] == 0:
            continue
        Gb = G_bias[li]                                          # [R][n]
        Gk = G_key[li] - beta * Gb[..., None] * refs[:, None, :]  # [R][n][d]
        Gs = w * (np.einsum("rnd,rncd->rnc", Gk, ck) - np.einsum("rnd,rnd->rn", Gk, key)[..., None] + Gb[..., None])
        grad += beta * (np.einsum("rnc,rncd->rd", Gs, ck) - np.einsum("rn,rnd->rd", Gb, key))
        if li > 0:
            n = key.shape[1]
            Gc = w[..., None] * Gk[:, :, None, :] + beta * Gs[..., None] * refs[:, None, None, :]
            G_key[li - 1][:, : n * C] += Gc.reshape(R, n * C, d)
            G_bias[li - 1][:, : n * C] += Gs.reshape(R, n * C)
    return loss, grad
