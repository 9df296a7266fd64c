"""Checks c_abi_check.cu's outputs against the oracle: the MXFP4 quantizer bit
for bit, everything else with the parity tolerance of tests/parity_util.py.

    python tests/c_abi/compare.py <input dir> <output dir>
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "..", ".."))
sys.path.insert(0, os.path.join(HERE, ".."))
import oracle  # noqa: E402
from oracle import backward as bw  # noqa: E402
from parity_util import errors, REL_MAX, MAE_RMS  # noqa: E402

D, O = sys.argv[1].rstrip("/") + "/", sys.argv[2].rstrip("/") + "/"
def rd(p, dt, shape): return np.fromfile(p, dtype=dt).reshape(shape)
ok = True
def check(name, y, ref):
    global ok
    rel, mae = errors(y, ref)
    good = rel <= REL_MAX and mae <= MAE_RMS and np.all(np.isfinite(y))
    ok &= good
    print(f"{name:28s} rel_max={rel:.2e} mae/rms={mae:.2e} {'OK' if good else 'FAIL'}")
# 1. MXFP4 quantize bit-exact
W = rd(D + 'mx_W.bin', np.float32, (3, 256, 768))
p_ref, s_ref = oracle.quantize_mxfp4(W)
P = rd(O + 'mxq_P.bin', np.uint8, p_ref.shape); S = rd(O + 'mxq_S.bin', np.uint8, s_ref.shape)
eq = np.array_equal(P, p_ref) and np.array_equal(S, s_ref); ok &= eq
print("mxfp4_quantize bit-exact:", eq, "(packed mismatches", int((P != p_ref).sum()), "scale mismatches", int((S != s_ref).sum()), ")")
# 2. MXFP4 GEMV
E, N, K = 6, 384, 512
P2 = rd(D + 'mx_P.bin', np.uint8, (E, N, K // 2)); S2 = rd(D + 'mx_S.bin', np.uint8, (E, N, K // 32))
off = rd(D + 'mx_off.bin', np.int32, (E + 1,)); M = int(off[-1])
X = rd(D + 'mx_X.bin', np.float16, (M, K)).astype(np.float64)
ref = oracle.grouped_gemm_mxfp4(X, P2, S2, off)
check("mxfp4 gemv none", rd(O + 'mxg_none.bin', np.float32, (M, N)), ref)
check("mxfp4 gemv swiglu", rd(O + 'mxg_swiglu.bin', np.float32, (M, N // 2)), oracle.swiglu(ref))
# 3. gemm_t
for tag, (E, N, K) in (("gt", (4, 2048, 1024)), ("gt2", (4, 70, 320))):
    off = rd(D + f'{tag}_off.bin', np.int32, (E + 1,)); M = int(off[-1])
    P = rd(D + f'{tag}_P.bin', np.uint8, (E, N, K // 2)); A = rd(D + f'{tag}_A.bin', np.float32, (E, N * K // 64))
    G = np.fromfile(D + f'{tag}_G.bin', np.float32).reshape(-1, N)[:M].astype(np.float64)
    check(f"gemm_t {N}x{K}", rd(O + f'{tag}_out.bin', np.float32, (M, K)), bw.grouped_gemm_t(G, P, A, off))
# 4. swiglu backward
gu = rd(D + 'sb_gu.bin', np.float32, (37, 192)); dh = rd(D + 'sb_dh.bin', np.float32, (37, 96))
check("swiglu backward", rd(O + 'sb_out.bin', np.float32, (37, 192)), bw.swiglu_backward(gu, dh))
# 5. combine + route backward
T, E, k, H = 33, 16, 4, 256
lg = rd(D + 'cb_lg.bin', np.float32, (T, E)); Yp = rd(D + 'cb_Yp.bin', np.float32, (T * k, H)); dY = rd(D + 'cb_dY.bin', np.float32, (T, H))
for rn in (0, 1):
    idx, w = oracle.route_topk(lg, k, bool(rn)); _, _, inv = oracle.permute_by_expert(idx, E)
    rdYp, rdw = bw.combine_backward(dY, Yp, inv, w)
    check(f"combine bw dYp renorm={rn}", rd(O + f'cb_dYp{rn}.bin', np.float32, (T * k, H)), rdYp)
    check(f"combine bw dw renorm={rn}", rd(O + f'cb_dw{rn}.bin', np.float32, (T, k)), rdw)
    check(f"route bw renorm={rn}", rd(O + f'cb_dl{rn}.bin', np.float32, (T, E)), bw.route_backward(lg, idx, rdw, bool(rn)))
print("ALL OK" if ok else "SOME FAILED")
sys.exit(0 if ok else 1)
