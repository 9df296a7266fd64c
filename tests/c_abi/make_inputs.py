"""Inputs of c_abi_check.cu: seeded numpy arrays, quantized and routed by the
oracle only.  Shapes are fixed here and in c_abi_check.cu.

    python tests/c_abi/make_inputs.py <input dir>
"""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.join(os.path.dirname(os.path.abspath(__file__)), "..", ".."))
import oracle  # noqa: E402

rng = np.random.default_rng(123)
D = sys.argv[1]
os.makedirs(D, exist_ok=True)
def w(name, a):
    np.ascontiguousarray(a).tofile(os.path.join(D, name))
# 1. MXFP4 quantize input W [3, 256, 768] fp32
E1, N1, K1 = 3, 256, 768
W = (rng.standard_normal((E1, N1, K1)) * 0.02).astype(np.float32)
W[rng.random(W.shape) < 1e-3] *= 30
W[0, 3, :32] = 0; W[0, 1, 32:64] = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 4, np.float32)
W[0, 2, :32] = (rng.standard_normal(32) * 2.0 ** -135).astype(np.float32)
w('mx_W.bin', W)
# 2. MXFP4 GEMV: oracle-quantized weights [6, 384, 512], X [M, 512] fp16, ragged offsets
counts = [1, 0, 9, 16, 17, 40]; E2, N2, K2 = 6, 384, 512
off2 = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32); M2 = int(off2[-1])
W2 = (rng.standard_normal((E2, N2, K2)) * 0.03).astype(np.float32)
P2, S2 = oracle.quantize_mxfp4(W2)
X2 = rng.standard_normal((M2, K2)).astype(np.float16)
w('mx_P.bin', P2); w('mx_S.bin', S2); w('mx_X.bin', X2); w('mx_off.bin', off2)
# 3. transposed NF4 GEMM: [4, 2048, 1024] with counts [8, 8, 0, 40], G fp32 [M+2, 2048]
E3, N3, K3 = 4, 2048, 1024; c3 = [8, 8, 0, 40]
off3 = np.concatenate([[0], np.cumsum(c3)]).astype(np.int32); M3 = int(off3[-1])
W3 = (rng.standard_normal((E3, N3, K3)) * 0.05).astype(np.float32)
P3, A3 = oracle.quantize_blockwise(W3)
G3 = rng.standard_normal((M3 + 2, N3)).astype(np.float32)
w('gt_P.bin', P3); w('gt_A.bin', A3.reshape(E3, -1)); w('gt_G.bin', G3); w('gt_off.bin', off3)
# 3b. small odd case: [4, 70, 320] counts [1, 0, 9, 3]
E4, N4, K4 = 4, 70, 320; c4 = [1, 0, 9, 3]
off4 = np.concatenate([[0], np.cumsum(c4)]).astype(np.int32); M4 = int(off4[-1])
W4 = (rng.standard_normal((E4, N4, K4)) * 0.05).astype(np.float32)
P4, A4 = oracle.quantize_blockwise(W4)
G4 = rng.standard_normal((M4, N4)).astype(np.float32)
w('gt2_P.bin', P4); w('gt2_A.bin', A4.reshape(E4, -1)); w('gt2_G.bin', G4); w('gt2_off.bin', off4)
# 4. SwiGLU backward: gu [37, 192], dh [37, 96]
gu = (rng.standard_normal((37, 192)) * 3).astype(np.float32); dh = rng.standard_normal((37, 96)).astype(np.float32)
w('sb_gu.bin', gu); w('sb_dh.bin', dh)
# 5. combine + route backward: T 33, E 16, k 4, H 256, both renorm modes
T, E, k, H = 33, 16, 4, 256
lg = rng.standard_normal((T, E)).astype(np.float32)
Yp = rng.standard_normal((T * k, H)).astype(np.float32); dY = rng.standard_normal((T, H)).astype(np.float32)
w('cb_lg.bin', lg); w('cb_Yp.bin', Yp); w('cb_dY.bin', dY)
for rn in (0, 1):
    idx, wt = oracle.route_topk(lg, k, bool(rn))
    _, _, inv = oracle.permute_by_expert(idx, E)
    w(f'cb_idx{rn}.bin', idx.astype(np.int32)); w(f'cb_w{rn}.bin', wt.astype(np.float32)); w(f'cb_inv{rn}.bin', inv.astype(np.int32))
print("sizes", M2, M3, M4)
