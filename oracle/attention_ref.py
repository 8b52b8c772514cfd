"""fp64 CPU oracle for exact attention.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The CUDA library never calls it and it
shares no code with the CUDA library.

What it computes, and where that is defined:

* Forward: ``O = softmax(scale * Q K^T [+ causal mask]) V`` computed from the
  plain definition, with the N x N score matrix S and probability matrix P
  materialised.  The three-line "S = QK^T; P = softmax(S); O = PV" form is the
  one in "CUDA-kernel-level optimisation: why Flash Attention is 5-10x faster
  than native PyTorch" (guanweilu.cn), section "three lines of PyTorch"; the
  1/sqrt(D) scaling and the (B, H, N, D) layout are from ``naive_attention`` in
  "Flash Attention principles: making Transformers faster" (ijyty.com),
  section "memory bottleneck"; the max-subtracted softmax is that page's
  ``stable_softmax`` (section "numerical stability").
* The saved per-row statistic is the natural-log logsumexp
  ``lse_i = m_i + ln(l_i)`` of the scaled scores, with m the row max and l the
  row sum of exp(s - m).  The pages name only m and l ("LLM paper notes #8:
  FlashAttention" (adg.csdn.net), section "online softmax"); lse in natural
  log is the plainest reading of "logsumexp".
* Causal mask: top-left aligned, key j is allowed for query i iff j <= i
  (the pages do not define a mask; this is the usual lower-triangular one).
* Backward: the pages only say that P is recomputed instead of stored (section
  "recomputation" of the adg.csdn.net notes).  The gradients here are the
  textbook softmax calculus of the forward definition, with L a scalar loss and
  dO = dL/dO:
      dV = P^T dO,  dP = dO V^T,  Delta_i = sum_j P_ij dP_ij,
      dS = P * (dP - Delta),  dQ = scale * dS K,  dK = scale * dS^T Q.
* A second forward, ``attention_forward_online``, follows the tiled
  online-softmax steps (sections "tiling" and "online softmax" of the
  adg.csdn.net notes; section "three tricks" of the guanweilu.cn article;
  ``flash_attention_blocked`` of the ijyty.com page, read with the rescale
  factor the printed line drops: O <- exp(m - m_new) * O + P V_j on the
  unnormalised accumulator, normalised once at the end).
* ``attention_sampled_rows`` is the plain definition evaluated row by row for
  sequences too long to materialise N x N at once (rows in chunks; the chunk
  size changes only summation order, at the 1e-16 level).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, a hand-worked example under ``tests/golden/``, invariants,
brute force, central finite differences, and torch's own CPU attention as a
second witness).  No function is "parity unpinned".
"""
from __future__ import annotations

import math

import torch

F64 = torch.float64


def to_f64(x) -> torch.Tensor:
    """Decode any float tensor (bf16 / fp32 / fp64, CPU or not) exactly to fp64 on the CPU."""
    return x.detach().to("cpu").to(F64)


def _causal_mask(nq: int, nk: int, row0: int = 0, col0: int = 0) -> torch.Tensor:
    """Boolean mask, True where key (col0 + c) > query (row0 + r): those scores are removed."""
    r = torch.arange(nq).unsqueeze(1) + row0
    c = torch.arange(nk).unsqueeze(0) + col0
    return c > r


def _head_probs(q, k, scale, causal):
    """S = scale * q k^T (one head), masked, and its row statistics.

    Returns (P normalised, m row max, l row sum of exp(S - m))."""
    S = scale * (q @ k.transpose(0, 1))
    if causal:
        S = S.masked_fill(_causal_mask(S.shape[0], S.shape[1]), float("-inf"))
    m = S.max(dim=1, keepdim=True).values
    E = torch.exp(S - m)
    l = E.sum(dim=1, keepdim=True)
    return E / l, m, l


def attention_forward(q, k, v, scale: float, causal: bool):
    """Plain-definition forward.  q, k, v: (B, H, N, D).  Returns (O, lse) in fp64."""
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    B, H, N, D = q.shape
    O = torch.empty(B, H, N, v.shape[-1], dtype=F64)
    lse = torch.empty(B, H, N, dtype=F64)
    for b in range(B):
        for h in range(H):
            P, m, l = _head_probs(q[b, h], k[b, h], scale, causal)
            O[b, h] = P @ v[b, h]
            lse[b, h] = (m + torch.log(l)).squeeze(1)
    return O, lse


def attention_probs(q, k, scale: float, causal: bool):
    """The full probability tensor P (B, H, N, N), for invariant checks on small inputs."""
    q, k = to_f64(q), to_f64(k)
    B, H, N, _ = q.shape
    P = torch.empty(B, H, N, k.shape[2], dtype=F64)
    for b in range(B):
        for h in range(H):
            P[b, h] = _head_probs(q[b, h], k[b, h], scale, causal)[0]
    return P


def attention_backward(q, k, v, do, scale: float, causal: bool):
    """Plain-definition forward and analytic backward.

    Returns a dict with O, lse, Delta (= rowsum(P * dP) = rowsum(dO * O)), dQ, dK, dV, all fp64."""
    q, k, v, do = to_f64(q), to_f64(k), to_f64(v), to_f64(do)
    B, H, N, D = q.shape
    out = {name: torch.empty(B, H, N, D, dtype=F64) for name in ("O", "dQ", "dK", "dV")}
    out["lse"] = torch.empty(B, H, N, dtype=F64)
    out["Delta"] = torch.empty(B, H, N, dtype=F64)
    for b in range(B):
        for h in range(H):
            P, m, l = _head_probs(q[b, h], k[b, h], scale, causal)
            O = P @ v[b, h]
            dV = P.transpose(0, 1) @ do[b, h]
            dP = do[b, h] @ v[b, h].transpose(0, 1)
            Delta = (P * dP).sum(dim=1, keepdim=True)
            dS = P * (dP - Delta)
            out["O"][b, h] = O
            out["lse"][b, h] = (m + torch.log(l)).squeeze(1)
            out["Delta"][b, h] = Delta.squeeze(1)
            out["dV"][b, h] = dV
            out["dQ"][b, h] = scale * (dS @ k[b, h])
            out["dK"][b, h] = scale * (dS.transpose(0, 1) @ q[b, h])
    return out


def attention_forward_online(q, k, v, scale: float, causal: bool, block_m: int, block_n: int):
    """Tiled forward with the online softmax, in the pages' order of steps.

    For each block of block_m query rows, walk the key/value blocks of
    block_n rows keeping, per row, the running max m and running sum l; each
    new block raises m to m_new, rescales the earlier sum and the unnormalised
    output accumulator by exp(m - m_new), and adds its own exp(S - m_new) terms.
    After the last block the accumulator is divided by l once.
    Returns (O, lse) in fp64."""
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    B, H, N, D = q.shape
    Nk = k.shape[2]
    O = torch.empty(B, H, N, v.shape[-1], dtype=F64)
    lse = torch.empty(B, H, N, dtype=F64)
    for b in range(B):
        for h in range(H):
            for i0 in range(0, N, block_m):
                qi = q[b, h, i0:i0 + block_m]
                rows = qi.shape[0]
                m = torch.full((rows, 1), float("-inf"), dtype=F64)
                l = torch.zeros(rows, 1, dtype=F64)
                acc = torch.zeros(rows, v.shape[-1], dtype=F64)
                for j0 in range(0, Nk, block_n):
                    if causal and j0 > i0 + rows - 1:
                        break                      # every key of this block is masked
                    kj = k[b, h, j0:j0 + block_n]
                    vj = v[b, h, j0:j0 + block_n]
                    s = scale * (qi @ kj.transpose(0, 1))
                    if causal:
                        s = s.masked_fill(_causal_mask(rows, kj.shape[0], i0, j0), float("-inf"))
                    m_new = torch.maximum(m, s.max(dim=1, keepdim=True).values)
                    p = torch.exp(s - m_new)
                    alpha = torch.exp(m - m_new)
                    l = alpha * l + p.sum(dim=1, keepdim=True)
                    acc = alpha * acc + p @ vj
                    m = m_new
                O[b, h, i0:i0 + rows] = acc / l
                lse[b, h, i0:i0 + rows] = (m + torch.log(l)).squeeze(1)
    return O, lse


def attention_bruteforce(q, k, v, scale: float, causal: bool):
    """Scalar triple loop with math.exp, for tiny inputs only (a second, independent witness)."""
    q, k, v = to_f64(q).tolist(), to_f64(k).tolist(), to_f64(v).tolist()
    B, H, N, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Dv = len(v[0][0][0])
    O = [[[[0.0] * Dv for _ in range(N)] for _ in range(H)] for _ in range(B)]
    lse = [[[0.0] * N for _ in range(H)] for _ in range(B)]
    for b in range(B):
        for h in range(H):
            for i in range(N):
                keys = range(i + 1) if causal else range(N)
                s = {j: scale * sum(q[b][h][i][d] * k[b][h][j][d] for d in range(D)) for j in keys}
                mx = max(s.values())
                w = {j: math.exp(s[j] - mx) for j in keys}
                tot = sum(w.values())
                for d in range(Dv):
                    O[b][h][i][d] = sum(w[j] * v[b][h][j][d] for j in keys) / tot
                lse[b][h][i] = mx + math.log(tot)
    return torch.tensor(O, dtype=F64), torch.tensor(lse, dtype=F64)


def _row_stats_chunked(qh, kh, vh, doh, scale, causal, chunk):
    """Per-row lse and Delta = rowsum(dO * O) of one head, computed chunk of rows by chunk."""
    N = qh.shape[0]
    lse = torch.empty(N, dtype=F64)
    delta = torch.empty(N, dtype=F64)
    O = torch.empty(N, vh.shape[1], dtype=F64)
    for r0 in range(0, N, chunk):
        r1 = min(N, r0 + chunk)
        kend = r1 if causal else kh.shape[0]       # keys beyond the chunk's last row are all masked
        S = scale * (qh[r0:r1] @ kh[:kend].transpose(0, 1))
        if causal:
            S = S.masked_fill(_causal_mask(r1 - r0, kend, r0, 0), float("-inf"))
        m = S.max(dim=1, keepdim=True).values
        E = torch.exp(S - m)
        l = E.sum(dim=1, keepdim=True)
        Oc = (E @ vh[:kend]) / l
        O[r0:r1] = Oc
        lse[r0:r1] = (m + torch.log(l)).squeeze(1)
        delta[r0:r1] = (doh[r0:r1] * Oc).sum(dim=1)
    return O, lse, delta


def attention_sampled_rows(q, k, v, do, scale: float, causal: bool, q_rows, k_rows, chunk: int = 512,
                           heads=None):
    """Plain definition evaluated on sampled rows of long sequences.

    For each head: first every row's lse and Delta (needed by any key row's
    gradient), computed in chunks of query rows; then, on the sampled query rows,
    O, lse and dQ = scale * sum_j dS_ij k_j; and on the sampled key rows,
    dV_j = sum_i P_ij dO_i and dK_j = scale * sum_i dS_ij q_i, with
    P_ij = exp(s_ij - lse_i) and dS_ij = P_ij (dO_i . v_j - Delta_i).

    q_rows / k_rows: dict head-index -> 1-D index tensor (head index = b*H + h).
    Returns dict head-index -> dict(O, lse, dQ at q_rows; dK, dV at k_rows)."""
    B, H, N, D = q.shape
    results = {}
    for bh in (heads if heads is not None else range(B * H)):
        b, h = divmod(bh, H)
        qh, kh, vh = to_f64(q[b, h]), to_f64(k[b, h]), to_f64(v[b, h])
        doh = to_f64(do[b, h])
        O_all, lse_all, delta_all = _row_stats_chunked(qh, kh, vh, doh, scale, causal, chunk)
        qr = q_rows[bh].long()
        kr = k_rows[bh].long()
        # sampled query rows: dQ
        S = scale * (qh[qr] @ kh.transpose(0, 1))                       # (nq, N)
        if causal:
            S = S.masked_fill(torch.arange(N).unsqueeze(0) > qr.unsqueeze(1), float("-inf"))
        P = torch.exp(S - lse_all[qr].unsqueeze(1))
        dP = doh[qr] @ vh.transpose(0, 1)
        dS = P * (dP - delta_all[qr].unsqueeze(1))
        dQ = scale * (dS @ kh)
        # sampled key rows: dK, dV (column j of P and dS)
        St = scale * (kh[kr] @ qh.transpose(0, 1))                      # (nk, N): s_ij for j in kr
        if causal:
            St = St.masked_fill(torch.arange(N).unsqueeze(0) < kr.unsqueeze(1), float("-inf"))
        Pt = torch.exp(St - lse_all.unsqueeze(0))
        dPt = vh[kr] @ doh.transpose(0, 1)                              # dO_i . v_j
        dSt = Pt * (dPt - delta_all.unsqueeze(0))
        results[bh] = {
            "O": O_all[qr], "lse": lse_all[qr], "dQ": dQ,
            "dV": Pt @ doh, "dK": scale * (dSt @ qh),
        }
    return results


def attention_delta(o, do):
    """Delta_i = sum_d dO_id * O_id (fp64), the backward's per-row correction term."""
    return (to_f64(do) * to_f64(o)).sum(dim=-1)
