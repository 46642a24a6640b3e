"""The expert-parallel layer's steps on the CPU for host-logic tests on gloo ranks: selection,
experts and combine by the FP64 oracle, gathers by indexing. Test infrastructure only."""
import numpy as np
import torch

import oracle


class CpuOracleOps:
    device = "cpu"

    def tensor(self, a, dtype=None):
        return torch.as_tensor(np.asarray(a), dtype=dtype)

    def to_host(self, t):
        return t.numpy()

    def route(self, x, router_w, router_scale, T, d, E, k):
        xb = x.numpy().view(np.uint16)
        ids, w, _ = oracle.topk_softmax(oracle.router_logits(xb, router_w.numpy()), k,
                                        float(router_scale.numpy()[0]))
        return torch.from_numpy(ids), torch.from_numpy(w)

    def gather(self, src, index, n, row_elems):
        return src[index.long()].reshape(n, row_elems).contiguous()

    def experts(self, x_rows, e_rows, w_rows, gate_up, down, expert_scale, R, d, f, e_local):
        out = np.zeros((R, d), dtype=np.float64)
        xb = x_rows.numpy().view(np.uint16)
        gu, dn, es = gate_up.numpy(), down.numpy(), expert_scale.numpy()
        for r in range(R):
            e = int(e_rows[r])
            _, y = oracle.expert_ffn(xb[r], gu[e], dn[e], d, f)
            out[r] = float(w_rows[r]) * float(es[e]) * y
        return torch.from_numpy(out)

    def combine(self, y_slots, T, d, k):
        y = y_slots.numpy().reshape(T, k, d)
        out = np.zeros((T, d), dtype=np.float64)
        for j in range(k):
            out += y[:, j]
        return torch.from_numpy(out)
