"""Router oracle: softmax over all experts, top-k selection, and the backward of the
selected probabilities with respect to the logits -- TEST INFRASTRUCTURE ONLY.

Sources: "MoE-Training für biologische Grundmodelle optimieren" (hyper.ai), the passage
on token routing (a router assigns each token to experts before the expert MLP) and the
French page's description of the routed expert computation. The pages name the router
but fix no formula; the readings:
  * probabilities are a softmax over all E experts of the token's logits (no
    renormalisation over the selected k);
  * the k experts with the largest probabilities are selected, in descending order;
    softmax is monotone in the logit, so the order is that of the logits, and equal
    logits keep the lower expert index first;
  * a logit of -inf marks an expert the token may not use (probability 0).
The selection is a decision taken on the fp32 logits as given (exact comparisons), so
the GPU and this oracle decide identically; the probabilities are computed in fp64.
"""
import numpy as np


def softmax(logits):
    """P[t, e] = exp(l[t, e] - max_e l[t]) / sum_e exp(l[t, e] - max_e l[t]), fp64."""
    l = np.asarray(logits, dtype=np.float64)
    m = np.max(l, axis=1, keepdims=True)
    if not np.all(np.isfinite(m)):
        raise ValueError("every row needs a finite logit")
    ex = np.exp(l - m)
    return ex / np.sum(ex, axis=1, keepdims=True)


def topk(logits, k):
    """(idx int64[T, k], probs fp64[T, k]): the k largest logits per row, descending,
    ties to the lower expert index; probs are the softmax over all experts at idx."""
    l = np.asarray(logits, dtype=np.float32)
    T, E = l.shape
    if not 1 <= k <= E:
        raise ValueError("k out of range")
    p = softmax(l)
    idx = np.zeros((T, k), dtype=np.int64)
    for t in range(T):
        # sort key: larger logit first, then lower index (a stable sort on -l)
        order = sorted(range(E), key=lambda e: (-float(l[t, e]), e))
        idx[t] = order[:k]
    return idx, np.take_along_axis(p, idx, axis=1)


def topk_backward(logits, idx, dprobs):
    """dL/dlogits for L depending on the selected probabilities only:
    dl[t, e] = sum_j dprobs[t, j] * dP[t, idx[t, j]] / dl[t, e]
             = P[t, e] * (g[t, e] - sum_j dprobs[t, j] * P[t, idx[t, j]]),
    with g[t, e] = dprobs[t, j] where idx[t, j] = e (0 for unselected experts),
    from dP_i / dl_e = P_i * (delta_ie - P_e)."""
    p = softmax(logits)
    idx = np.asarray(idx, dtype=np.int64)
    d = np.asarray(dprobs, dtype=np.float64)
    T, E = p.shape
    g = np.zeros((T, E), dtype=np.float64)
    for t in range(T):
        for j in range(idx.shape[1]):
            g[t, idx[t, j]] += d[t, j]
    s = np.sum(g * p, axis=1, keepdims=True)
    return p * (g - s)
