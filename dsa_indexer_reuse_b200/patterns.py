"""Layer-overlap matrix and pattern search on a workload's inputs (a tool).

    python -m dsa_indexer_reuse_b200.patterns --workload prefill-8k --n-full 4

Runs every layer's own indexer (as with index_topk_freq = 1), measures the
pairwise top-k overlap of the layers' index sets on the GPU
(ic_topk_overlap), and prints the matrix, the pattern that maximises overlap
coverage for the requested number of Full layers (ic_search_pattern), and the
greedy pattern for the same count (ic_greedy_pattern) under either that
coverage or, with --objective attn-error, the stack's attention-output error
against the all-Full stack (a proxy for the pages' language-modelling loss,
which needs trained weights and calibration data).

On the synthetic Gaussian inputs of this package the layers are independent,
so the overlaps sit near k / (keys visible) and say nothing about a trained
model; on a trained model's indexer inputs the same calls give the pages'
Appendix Figure 4 style matrix.
"""

from __future__ import annotations

import argparse

import numpy as np
import torch

from . import workloads as W


def layer_overlap(wl, n_layers: int, seed: int = 0, device="cuda") -> np.ndarray:
    import dsa_indexer_reuse_b200 as ic
    idx = []
    for layer in range(n_layers):
        ind = W.indexer_inputs(wl, layer, seed=seed, device=device)
        idx.append(ic.indexer_topk(ind["q_I"], ind["w"], ind["k_I"], wl.topk, q_scale=ind["q_scale"],
                                   k_scale=ind["k_scale"], q_pos0=wl.q_pos0))
    return ic.overlap_matrix(idx, wl.n_k)


def attention_error_objective(wl, n_layers: int, seed: int = 0, device="cuda"):
    """objective(pattern) = relative L2 error of every layer's attention output
    against the all-Full stack, on the workload's seeded inputs."""
    import dsa_indexer_reuse_b200 as ic
    layers = []
    for l in range(n_layers):
        d = dict(W.indexer_inputs(wl, l, seed=seed, device=device))
        d.update(W.attention_inputs(wl, l, seed=seed, device=device))
        d["out"] = torch.empty((wl.batch, wl.n_q, wl.H, wl.d_v), dtype=torch.bfloat16, device=device)
        layers.append(d)
    shape = dict(batch=wl.batch, n_q=wl.n_q, n_k=wl.n_k, q_pos0=wl.q_pos0, H_I=wl.H_I, d_I=wl.d_I,
                 topk=wl.topk, qk_dtype=wl.qk_dtype, w_dtype=wl.w_dtype, H=wl.H, d_qk=wl.d_qk,
                 d_v=wl.d_v, sm_scale=wl.sm_scale)
    ic.layer_stack(layers, shape, pattern="F" * n_layers)
    ref = [L["out"].float().clone() for L in layers]
    ref_norm = sum(float(r.norm()) ** 2 for r in ref) ** 0.5

    def objective(pattern: str) -> float:
        ic.layer_stack(layers, shape, pattern=pattern)
        err = sum(float((L["out"].float() - r).norm()) ** 2 for L, r in zip(layers, ref)) ** 0.5
        return err / max(ref_norm, 1e-30)

    return objective


def main(argv=None):
    import dsa_indexer_reuse_b200 as ic
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="tiny-int", choices=sorted(W.WORKLOADS))
    ap.add_argument("--layers", type=int, default=0, help="layers to measure (default: the workload's)")
    ap.add_argument("--seq-len", type=int, default=0, help="override n_q = n_k")
    ap.add_argument("--n-full", type=int, default=0, help="Full layers of the searched pattern")
    ap.add_argument("--objective", default="coverage", choices=["coverage", "attn-error"],
                    help="objective of the greedy search")
    args = ap.parse_args(argv)
    wl = W.WORKLOADS[args.workload]
    if args.seq_len:
        wl = wl.with_(n_q=args.seq_len, n_k=args.seq_len)
    n = args.layers or wl.n_layers
    R = layer_overlap(wl, n)
    torch.cuda.synchronize()
    np.set_printoptions(precision=3, suppress=True, linewidth=200)
    print("overlap ratio R[a][b] = |T_a & T_b| / |T_a| over all rows, %d layers of %s" % (n, wl.name))
    print(R)
    n_full = args.n_full or max(1, n // 4)
    pat, score = ic.search_pattern(R, n_full)
    print("searched pattern (n_full=%d): %s  coverage %.4f of %d" % (n_full, pat, score, n))
    if args.objective == "coverage":
        gpat, gval = ic.greedy_pattern(n, n_full, lambda p: -ic.pattern_score(R, p))
        print("greedy pattern   (n_full=%d): %s  coverage %.4f of %d" % (n_full, gpat, -gval, n))
    else:
        gpat, gval = ic.greedy_pattern(n, n_full, attention_error_objective(wl, n))
        print("greedy pattern   (n_full=%d): %s  attention-output error %.4g vs all-Full" % (n_full, gpat, gval))


if __name__ == "__main__":
    main()
