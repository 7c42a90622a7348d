"""The expert-parallel layer's kernel calls, written with the oracle on CPU
tensors, so the layer's exchange and bookkeeping run as gloo ranks on CPU.

Same call signatures as the library's moe_ep_dispatch / moe_ep_expert_ffn /
moe_ep_combine; each step is the oracle's: routing and permutation, one expert
row at a time (rounded to bf16, as the GPU stores its expert outputs), the
shared expert and the combine in slot order."""
import numpy as np
import torch

import oracle


def _bf16(a64):
    """fp64 array -> bf16 torch tensor (round to nearest even)."""
    bits = oracle.f64_to_bf16(np.ascontiguousarray(a64, dtype=np.float64))
    return torch.from_numpy(bits.astype(np.uint16).view(np.int16)).view(torch.bfloat16)


def _f64(t):
    return t.to(torch.float32).numpy().astype(np.float64)


def _u16(t):
    return np.ascontiguousarray(t.contiguous().view(torch.int16).numpy().view(np.uint16))


class OracleOps:
    @staticmethod
    def moe_ep_dispatch_workspace_size(T, d, E, k):
        return 0

    @staticmethod
    def moe_ep_expert_ffn_workspace_size(rows, d, R, E_local, inter):
        return 0

    @staticmethod
    def moe_ep_combine_workspace_size(T, d, inter):
        return 0

    @staticmethod
    def moe_ep_dispatch(x, w_router, bias, k, scale, topk_idx, topk_w, counts, slot_row,
                        send_rows, workspace):
        E = w_router.shape[0]
        ridx, rw, _ = oracle.route(x, w_router, bias, k, scale)
        cnt, _, row_token, sr = oracle.permute(ridx, E)
        topk_idx.copy_(torch.from_numpy(ridx))
        topk_w.copy_(torch.from_numpy(rw.astype(np.float32)))
        counts.copy_(torch.from_numpy(cnt.astype(np.int32)))
        slot_row.copy_(torch.from_numpy(sr))
        send_rows.copy_(x[torch.from_numpy(row_token.astype(np.int64))])

    @staticmethod
    def moe_ep_expert_ffn(recv_rows, recv_counts, w_gate_up, w_down, y, workspace):
        R, El = recv_counts.shape
        cnt = recv_counts.numpy()
        row = 0
        for s in range(R):              # received rows: source-major, then local expert
            for e in range(El):
                gu, dn = _u16(w_gate_up[e]), _u16(w_down[e])
                for _ in range(int(cnt[s, e])):
                    y[row] = _bf16(oracle.swiglu_row(_u16(recv_rows[row]), gu, dn))
                    row += 1
        assert row == recv_rows.shape[0]

    @staticmethod
    def moe_ep_combine(y_back, x, ws_gate_up, ws_down, topk_w, slot_row, out, workspace):
        T = x.shape[0]
        gu, dn = _u16(ws_gate_up), _u16(ws_down)
        ysh = np.stack([oracle.swiglu_row(_u16(x[t]), gu, dn) for t in range(T)])
        o = oracle.combine(_f64(y_back), ysh, topk_w.numpy().astype(np.float64), slot_row.numpy())
        out.copy_(_bf16(o))
