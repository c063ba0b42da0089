"""The device steps of an expert-parallel pass done by the CPU oracle, so the
exchange logic (planning, both all-to-alls, regrouping, merge) can run as gloo
ranks on the CPU.  Test infrastructure only."""
import numpy as np
import torch

from oracle import moe_oracle as orc


class OracleOps:
    y_dtype = torch.float64

    def __init__(self, k: int, scale: float):
        self.k, self.scale = k, scale

    def route(self, h, Wr, bias, d):
        logits = orc.router_logits(h.float().numpy(), Wr.numpy())
        idx, w = orc.route(logits, bias.numpy(), self.k, self.scale)
        return torch.from_numpy(idx.astype(np.int32)), torch.from_numpy(w)

    def permute(self, idx, d):
        counts, offsets, perm, inv = orc.group_by_expert(idx.numpy(), d.E)
        return (torch.from_numpy(counts), torch.from_numpy(offsets), torch.from_numpy(perm),
                torch.from_numpy(inv))

    def gather_rows(self, src, idx, n_rows):
        return src[idx.long()] if n_rows else src[:0].clone()

    def expert_ffn(self, x, perm, offsets, W1, W3, W2, D, F):
        y = torch.zeros((x.shape[0], D), dtype=torch.float64)
        xf = x.float().numpy()
        off = offsets.numpy()
        p = perm.numpy()
        for e in range(W1.shape[0]):
            if off[e + 1] > off[e]:
                rows = p[off[e]:off[e + 1]]
                y[off[e]:off[e + 1]] = torch.from_numpy(orc.swiglu_expert(
                    xf[rows], W1[e].double().numpy(), W3[e].double().numpy(),
                    W2[e].double().numpy()))
        return y

    def shared_ffn(self, h, Ws1, Ws3, Ws2, y_full, routed_rows):
        T = h.shape[0]
        hf = h.float().numpy()
        for s in range(Ws1.shape[0]):
            y_full[routed_rows + s * T: routed_rows + (s + 1) * T] = torch.from_numpy(
                orc.swiglu_expert(hf, Ws1[s].double().numpy(), Ws3[s].double().numpy(),
                                  Ws2[s].double().numpy()))

    def combine(self, y_full, w, inv, d):
        T, k, S = d.T, d.k, d.S
        y = y_full.numpy()
        ysh = y[T * k:].reshape(S, T, -1) if S else None
        return torch.from_numpy(orc.combine(y[:T * k], w.numpy(), inv.numpy(), ysh))
