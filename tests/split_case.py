"""A small call for the head-split test: 5 heads, d = 64, a few key blocks
per row, and the oracle path over a range of its heads."""
import numpy as np

import oracle
from image_dits_b200.workload import Workload, make_qkv

SPLIT_WL = Workload("split", 1, 5, 64, 2, 8, 12, 2, 4, 4, 0.4, True, (24, 20, 20))


def _bits(x):
    return x.contiguous().view(dtype=__import__("torch").int16).numpy().view(np.uint16)


def oracle_call(wl, h0, h1):
    """Heads [h0, h1) of the call's inputs (seed 5) through the oracle:
    permutation (section 3.3), top-n block mask (section 3.2), masked
    attention (section 3.1), inverse permutation; float64 [B, h1-h0, N, d]."""
    q, k, v = (x[:, h0:h1].contiguous() for x in make_qkv(wl, "cpu", seed=5))
    perm = oracle.permutation(wl.frames, wl.height, wl.width, wl.win_t, wl.win_h, wl.win_w, wl.sink, wl.text_tokens)
    qp, kp, vp = (oracle.permute(_bits(x), perm) for x in (q, k, v))
    mask, _, _ = oracle.predict_mask(qp, kp, wl.keep, wl.frames, wl.height, wl.width, wl.sink, wl.text_tokens)
    op, _ = oracle.full_attention_output(qp, kp, vp, mask)      # float64 [B*(h1-h0), N, d]
    o = np.empty_like(op)
    o[:, perm, :] = op                                           # token at position p came from perm[p]
    return o.reshape(wl.batch, h1 - h0, wl.num_tokens, wl.head_dim)
