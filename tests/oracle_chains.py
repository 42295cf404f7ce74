"""Expected values built from oracle calls alone (test infrastructure), for
checks whose reference needs a whole column of the error estimate: every
oracle input here comes from the seeded generators or from other oracle
calls, never from the GPU."""
import numpy as np
import torch


def weight_rows(orc, c_or_r, is_r, d_out, offsets, gamma, seed, layer, draw_begin, K_total, sigma, X, rows,
                bf16=True, token_begin=0):
    """Rows `rows` of G_W = sum_t g_t x_t^T, with g_t[rows] from the oracle's
    estimate over every token.  g is taken to binary32 and, for the bf16
    weight GEMM, rounded to bf16 (nearest, ties to even): the precisions in
    which the kernels hold it before the GEMM, so both sides make the same
    rounding decisions up to binary32 ties."""
    T = np.asarray(c_or_r).shape[1]
    rows = np.asarray(rows)
    if not is_r:
        # one scan of every draw (the oracle's recurrence), held in binary32 as
        # the kernels hold r, instead of one recurrence per token
        c_or_r = orc.reward_scan(c_or_r, offsets, gamma).astype(np.float32)
    g = orc.layer_estimate(c_or_r, True, d_out, offsets, gamma, seed, layer, draw_begin, K_total, sigma,
                           np.arange(T), chans=rows, token_begin=token_begin).astype(np.float32)
    if bf16:
        # round to nearest bf16, ties to even (torch's CPU conversion)
        g = torch.from_numpy(g).to(torch.bfloat16).float().numpy()
    return orc.weight_grad(g, X, rows=np.arange(len(rows)))
