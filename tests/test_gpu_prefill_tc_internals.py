"""White-box check of the tensor-core prefill's first stage: the per-(chunk, head) workspace
records (W, Q~, K~, U, P, g_cum) written by the prep kernel, decoded from their operand layouts and
compared with a float64 evaluation of the chunk formulas on the same fp16 inputs. Localises a
failure to the prep or the scan stage."""
import numpy as np
import pytest
import torch

import synthetic
from gated_deltanet_linear_19_b200 import chunked_prefill, device_status, prefill_workspace_size
from tests.gpu_util import dims_of, make_layer, t_bits, t_f32, t_i32

pytestmark = pytest.mark.gpu

REC = 73984


def _decode_kmajor(buf, rows, cols, sbo):
    out = np.empty((rows, cols), np.float16)
    h = buf.view(np.float16)
    for r in range(rows):
        for k in range(cols):
            off = (r % 8) * 16 + (k % 8) * 2 + (r // 8) * sbo + (k // 8) * 128
            out[r, k] = h[off // 2]
    return out


def _decode_mnmajor(buf, m_rows, k_cols, sbo):
    """[k][m] view of an MN-major canonical operand (M contiguous inside a core matrix)."""
    out = np.empty((k_cols, m_rows), np.float16)
    h = buf.view(np.float16)
    for k in range(k_cols):
        for m in range(m_rows):
            off = (m % 8) * 2 + (k % 8) * 16 + (m // 8) * sbo + (k // 8) * 128
            out[k, m] = h[off // 2]
    return out


def test_prep_records_match_chunk_formulas():
    lengths = [100]
    w = synthetic.packed(lengths, seed=701, H_k=1, H_v=2, n_slots=1, conv_std=1.0)
    # slow decay (g of about -0.03 per token) keeps exp(g_cum) inside the fp16 range, so the
    # records are compared element by element rather than lost to underflow
    w["A_log"] = np.zeros_like(w["A_log"])
    w["dt_bias"] = np.full_like(w["dt_bias"], -4.0)
    dims = dims_of(w)
    layer = make_layer(w)
    T = 100
    q, k, v, g, beta = layer._front_bufs(T, torch.float16)
    from gated_deltanet_linear_19_b200 import conv_step
    conv_step(dims, t_bits(w["x"]), layer.conv_w, layer.conv_state, t_i32(w["cu_seqlens"]),
              t_i32(w["slot_ids"]), t_f32(w["a"]), t_f32(w["b"]), layer.A_log, layer.dt_bias,
              q, k, v, g, beta, eps=w["eps"], q_scale=w["q_scale"])
    need = prefill_workspace_size(dims, T, 1, 64, torch.float16)
    assert need > 0
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    o = torch.empty((T, 2, 128), dtype=torch.bfloat16, device="cuda")
    chunked_prefill(dims, q, k, v, g, beta, layer.state, t_i32(w["slot_ids"]),
                    t_i32(w["cu_seqlens"]), o, chunk=64, workspace=ws)
    assert device_status() == 0
    wsb = ws.cpu().numpy()
    qn, kn, vn = (t.cpu().double().numpy() for t in (q, k, v))
    gn, bn = g.cpu().double().numpy(), beta.cpu().double().numpy()
    for c, (c0, L) in enumerate([(0, 64), (64, 36)]):
        for h in range(2):
            rec = wsb[(c * 2 + h) * REC:(c * 2 + h + 1) * REC]
            K = np.zeros((64, 128)); Q = np.zeros((64, 128)); V = np.zeros((64, 128))
            K[:L] = kn[c0:c0 + L, 0]; Q[:L] = qn[c0:c0 + L, 0]; V[:L] = vn[c0:c0 + L, h]
            gg = np.zeros(64); bb = np.zeros(64)
            gg[:L] = gn[c0:c0 + L, h]; bb[:L] = bn[c0:c0 + L, h]
            gc = np.cumsum(gg)
            dec = np.exp(np.tril(gc[:, None] - gc[None, :]))
            Lm = np.tril(bb[:, None] * (K @ K.T) * dec, -1)
            Tm = np.linalg.inv(np.eye(64) + Lm)
            W = Tm @ (K * (bb * np.exp(gc))[:, None])
            U = Tm @ (V * bb[:, None])
            P = np.tril(Q @ K.T * dec)
            Qt = Q * np.exp(gc)[:, None]
            Kt = K * np.exp(gc[-1] - gc)[:, None]
            got_gc = rec[73728:73984].view(np.float32)
            np.testing.assert_allclose(got_gc, gc, rtol=1e-5, atol=1e-5)
            got_W = _decode_kmajor(rec[0:16384], 64, 128, 2048).astype(np.float64)
            got_Qt = _decode_kmajor(rec[16384:32768], 64, 128, 2048).astype(np.float64)
            got_Kt = _decode_mnmajor(rec[32768:49152], 128, 64, 1024).astype(np.float64)
            # U is stored as 4 column tiles of 32 columns, each an MN-major operand
            # (N = column, K = token; LBO 128, SBO 1024)
            got_U = np.concatenate(
                [_decode_mnmajor(rec[57344 + 4096 * j:57344 + 4096 * (j + 1)], 32, 64, 1024)
                 for j in range(4)], axis=1).astype(np.float64)
            got_P = _decode_kmajor(rec[49152:57344], 64, 64, 1024).astype(np.float64)
            errs = {}
            for name, got, ref in (("W", got_W, W), ("U", got_U, U), ("P", got_P, P),
                                   ("Q~", got_Qt, Qt), ("K~", got_Kt, Kt)):
                errs[name] = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
            print(f"chunk {c} head {h}: rel errors {errs}; |W|={np.linalg.norm(W):.3e} "
                  f"|got W|={np.linalg.norm(got_W):.3e} nonzero={np.count_nonzero(got_W)}")
            if errs["W"] > 3e-3:
                print("got W[0:2,0:8]", got_W[0:2, 0:8], "\nref W[0:2,0:8]", W[0:2, 0:8])
                raw = rec[0:16384].view(np.float16).astype(np.float64)
                print("raw W record nonzero:", np.count_nonzero(raw), raw[:16])
            assert all(e < 3e-3 for e in errs.values()), (c, h, errs)
