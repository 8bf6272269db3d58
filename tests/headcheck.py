"""Shared GPU-vs-oracle checks of whole head calls (imported by the -m gpu test files).

check_head runs one fused head call through the C ABI with debug outputs and compares it with the
oracle on the same inputs under the rules of parity.py:
  * probe sets bit-exact unless the oracle's p-th-cluster margin is within 4e-3 (then the clusters
    that differ must lie within 4e-3 of the threshold);
  * where the sets agree: candidate token ids bit-exact in slot order and candidate logits within
    2e-3 (debug="full");
  * tokens identical where the sets agree and the oracle's top-1 margin exceeds 4e-3, otherwise a
    near-maximum of the oracle's decision keys over the candidates the GPU used.
debug="sel" asks for the probe sets only, which keeps batched BF16 calls on the tensor-core path
(the per-candidate outputs exist only on the CUDA-core Stage 2)."""

import numpy as np
import torch

from clustered_retrieval_classification_b200 import synth
from parity import LOGIT_TOL, check_sets, check_tokens

DEV = "cuda"


def dev(a, kind):
    from clustered_retrieval_classification_b200 import flashhead as F
    return F.device_array(a, kind, DEV)


def load(fh, idx, int4=False, cluster_major=True):
    return fh.index_from_host(idx.E, idx.C, idx.C2T, idx.cfg.dtype, idx.C_q4, idx.C_scales,
                              int4=int4, cluster_major=cluster_major)


def run_head(fh, I, Hd, p, sample, tau, seed, step, P, B, debug="full"):
    dbg = dict(sel=torch.empty((B, p), dtype=torch.int32, device=DEV))
    if debug == "full":
        dbg.update(cand_tok=torch.empty((B, P), dtype=torch.int32, device=DEV),
                   cand_logit=torch.empty((B, P), dtype=torch.float32, device=DEV))
    if sample:
        tok = fh.head_sample(I, Hd, p, tau, seed, step, debug=dbg)
    else:
        tok = fh.head_greedy(I, Hd, p, debug=dbg)
    torch.cuda.synchronize()
    return tok.cpu().numpy(), {k: v.cpu().numpy() for k, v in dbg.items()}


def check_head(fh, orc, idx, H, p, sample=False, tau=1.0, seed=0, step=0, batch=None,
               cluster_major=True, int4=False, debug="full", I=None):
    """Returns (queries whose sets differ, queries whose tokens differ), all within the rules."""
    cfg = idx.cfg
    if I is None:
        I = load(fh, idx, int4=int4, cluster_major=cluster_major)
    B = batch or H.shape[0]
    Hq = H[:B]
    P = p * cfg.b
    tok, dbg = run_head(fh, I, dev(Hq, cfg.dtype), p, sample, tau, seed, step, P, B, debug)
    o = orc.head(idx, Hq, p, sample=sample, tau=tau, seed=seed, step=step, use_int4=int4)
    s = orc.stage1_scores(idx.C if not int4 else None, cfg.dtype, Hq, cfg.c, cfg.d,
                          q4=idx.C_q4 if int4 else None, scales=idx.C_scales if int4 else None)
    keys = orc.gumbel_keys(s, tau, seed, step, 0) if sample else s
    n_set = check_sets(dbg["sel"], o["sel"], keys, o["set_margin"])
    same = [set(dbg["sel"][q]) == set(o["sel"][q]) for q in range(B)]
    cand_gpu = dbg.get("cand_tok")
    if cand_gpu is None:  # the candidates of the GPU's own probe sets, in slot order
        cand_gpu = orc.gather(idx.C2T, dbg["sel"])
    for q in range(B):
        if same[q] and debug == "full":
            assert np.array_equal(dbg["cand_tok"][q], o["cand"][q])
            assert np.abs(dbg["cand_logit"][q] - o["z"][q]).max() <= LOGIT_TOL

    def valid(q, t):
        cand = cand_gpu[q:q + 1]
        z = orc.logits(idx.E, cfg.dtype, Hq[q:q + 1], cand)[0]
        if sample:
            g = np.array([orc.gumbel(orc.draw_u32(seed, step, q, 1, int(u))) for u in cand[0]])
            z = z / tau + g
        return z.max(), z[list(cand[0]).index(t)]

    n_tok = check_tokens(tok, o["tok"], o["tok_margin"], same, valid)
    return n_set, n_tok


def decided(o, gpu_sel, margin=4e-3):
    """Queries whose token the comparison rules decide: the GPU's probe set equals the oracle's and
    the oracle's top-1 margin exceeds `margin`."""
    return np.array([set(gpu_sel[q].tolist()) == set(o["sel"][q].tolist()) and
                     o["tok_margin"][q] > margin for q in range(len(o["tok"]))])


__all__ = ["dev", "load", "run_head", "check_head", "decided", "synth"]
