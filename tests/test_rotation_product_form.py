"""The product form of the rotation used by the GPU path for batches above 64
rows, checked on the CPU with the float64 oracle (GPTQModel wiki page
"ParoQuant", "Pairwise Givens rotations" and "Activation and weight
transforms"):

* each 128-channel group's stages with its channel scales are one linear map,
  x_g -> x_g R'_g with R'_g = diag(cs_g) G_0 ... G_{krot-1}, and row r of R'_g
  is the basis vector e_r scaled by cs[r] and taken through the stages — so
  rotating scaled basis rows and multiplying reproduces the stage-by-stage
  rotation;
* R'_g stored as two fp16 parts (hi = fp16(R'), lo = fp16(R' - hi)) keeps the
  product far inside the 1e-3 bound on X_r, where a single fp16 R' would not
  (outlier channels make some groups' entries large and the fp16 rounding of
  R' then shows in their small neighbours)."""
import numpy as np

import oracle
import synth

G = 128


def basis_rows(K):
    """[128, K]: row r has a one at channel g*128 + r of every group g, so one
    rotation of these rows yields every group's R'_g side by side."""
    E = np.zeros((G, K))
    for g in range(K // G):
        E[:, g * G:(g + 1) * G] = np.eye(G)
    return E


def product_form(x, Rstack, K):
    """x_g @ R'_g for every group g (float64)."""
    out = np.empty((x.shape[0], K))
    for g in range(K // G):
        sl = slice(g * G, (g + 1) * G)
        out[:, sl] = np.asarray(x, np.float64)[:, sl] @ Rstack[:, sl]
    return out


def rel_err(got, ref):
    rms = np.sqrt(np.mean(ref * ref, axis=1, keepdims=True))
    return float(np.max(np.abs(got - ref) / np.maximum(np.abs(ref), rms)))


def test_product_form_equals_stages():
    for krot, active in ((8, None), (1, None), (17, None), (8, 6)):
        lay = synth.make_layer("pf", 512, 32, seed=100 + krot, krot=krot, active_pairs=active, n_outliers=5)
        x = synth.make_activations(lay, 37)
        R = oracle.rotate(basis_rows(512), lay.channel_scales, lay.pairs, lay.theta, G, krot=krot)
        ref = oracle.rotate(x, lay.channel_scales, lay.pairs, lay.theta, G, krot=krot)
        assert rel_err(product_form(x, R, 512), ref) <= 1e-12


def test_scaling_only_product_is_diagonal():
    lay = synth.make_layer("pd", 256, 32, seed=7)
    R = oracle.rotate(basis_rows(256), lay.channel_scales, None, None, G, krot=0)
    for g in range(2):
        blk = R[:, g * G:(g + 1) * G]
        assert np.array_equal(blk, np.diag(np.asarray(lay.channel_scales, np.float64)[g * G:(g + 1) * G]))


def test_fp16_hi_lo_parts_keep_the_rotation_bound():
    lay = synth.make_layer("pp", 1024, 32, seed=11, n_outliers=10)
    x = synth.make_activations(lay, 256)
    R = oracle.rotate(basis_rows(1024), lay.channel_scales, lay.pairs, lay.theta, G)
    ref = oracle.rotate(x, lay.channel_scales, lay.pairs, lay.theta, G)
    R32 = R.astype(np.float32)                      # the parts are split from an fp32 build
    hi = R32.astype(np.float16)
    lo = (R32 - hi.astype(np.float32)).astype(np.float16)
    split = rel_err(product_form(x, hi.astype(np.float64) + lo.astype(np.float64), 1024), ref)
    single = rel_err(product_form(x, hi.astype(np.float64), 1024), ref)
    assert split <= 1e-5                            # 100x inside the 1e-3 bound on X_r
    assert single > 10 * split                      # the lo part is what buys it
