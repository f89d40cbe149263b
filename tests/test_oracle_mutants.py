"""The oracle's pins catch plausible mistakes.

Each case copies the oracle to a temporary directory, plants one slip in the
C source or in its Python layer by a textual substitution (a wrong sign, a
transposed U, a wrong bit position, a dropped term, another rounding, another
tie rule), builds it, and runs the pins of test_oracle_pins.py against that
copy: at least one pin must fail.  The real oracle is never modified.
Everything runs on the CPU.
"""

import importlib.util
import os
import shutil
import sys
import uuid

import pytest

import oracle as real_oracle
import test_oracle_pins as pins

SRC_DIR = os.path.dirname(real_oracle.__file__)

# (name, original text, planted text)
MUTANTS = [
    ("correction-sign", "s[j] = sm_scale * (base + sigma * corr);",
     "s[j] = sm_scale * (base - sigma * corr);"),
    ("projection-U-transposed", "const float term = U[(size_t)c * r + i] * e[c];",
     "const float term = U[(size_t)i * d + c] * e[c];"),
    ("projection-fused", "y[i] = y[i] + term;",
     "y[i] = fmaf(U[(size_t)c * r + i], e[c], y[i]);"),
    ("read-U-transposed",
     "acc += (double)U[(size_t)c * r + i] * zhat[(size_t)j * r + i];",
     "acc += (double)U[(size_t)i * d + c] * zhat[(size_t)j * r + i];"),
    ("residual-sign", "for (int c = 0; c < d; ++c) e[c] = x[c] - khat[c];",
     "for (int c = 0; c < d; ++c) e[c] = khat[c] - x[c];"),
    ("packing-order", "packed[ch >> 2] |= (uint8_t)(code << (2 * (ch & 3)));",
     "packed[ch >> 2] |= (uint8_t)(code << (2 * (3 - (ch & 3))));"),
    ("round-half-up", "const float t = nearbyintf(off / s);",
     "const float t = floorf(off / s + 0.5f);"),
    ("scale-by-reciprocal", "const float s = span / 3.0f;",
     "const float s = span * (1.0f / 3.0f);"),
    ("side-levels-8", "const float s = a / 7.0f;", "const float s = a / 8.0f;"),
    ("dropped-minimum", "xhat[c] = minimum[g] + prod;", "xhat[c] = prod;"),
    ("kl-sign", "kl[bh] = e1 - L + Lh;", "kl[bh] = e1 + L - Lh;"),
    ("variance-without-mean", "fvar[bh] = m2 - m1 * m1;", "fvar[bh] = m2;"),
    ("a2-weight-p", "a2 += p * p * n2;", "a2 += p * n2;"),
    ("head-to-kv-mapping", "const int kv = h / G;\n                    const int Tb = seq_lens ? seq_lens[b] : T;\n                    const size_t row = (size_t)b * Hkv + kv;",
     "const int kv = h % Hkv;\n                    const int Tb = seq_lens ? seq_lens[b] : T;\n                    const size_t row = (size_t)b * Hkv + kv;"),
    ("nibble-unsigned", "return v >= 8 ? v - 16 : v;", "return v;"),
    ("side-code-no-clamp", "w = t < -7.0f ? -7 : (t > 7.0f ? 7 : (int)t);",
     "w = (int)t;"),
    ("base-code-no-clamp", "code = t < 0.0f ? 0 : (t > 3.0f ? 3 : (int)t);",
     "code = (int)t;"),
    ("group-of-16", "static int group_size(int d) { return d < 32 ? d : 32; }",
     "static int group_size(int d) { return d < 16 ? d : 16; }"),
    # the per-channel base code
    ("channel-minimum-is-maximum", "            if (v < lo) lo = v;", "            if (v > lo) lo = v;"),
    ("channel-dequant-drops-minimum", "                xhat[(sq * T + t) * d + c] = mn[c] + prod;",
     "                xhat[(sq * T + t) * d + c] = prod;"),
]

# slips in the Python layer of the oracle (oracle/__init__.py)
MUTANTS_PY = [
    ("merge-equal-weights", "w = np.where(np.isfinite(lses), np.exp(lses - M0), 0.0)",
     "w = np.where(np.isfinite(lses), 1.0, 0.0)"),
    ("merge-lse-without-log", "lse = np.where(covered, M0 + np.log(L1), -np.inf)",
     "lse = np.where(covered, M0 + L1, -np.inf)"),
    ("a2-p-not-squared", "out[b, kv, :Tb] = (p * p).sum(axis=0) * dv2",
     "out[b, kv, :Tb] = p.sum(axis=0) * dv2"),
    ("a2-ties-to-higher-position", "order = sorted(range(Tb), key=lambda j: (-scores[b, kv, j], j))",
     "order = sorted(range(Tb), key=lambda j: (-scores[b, kv, j], -j))"),
    ("a2-kept-unsorted", "kept = sorted(order[:min(K, Tb)])", "kept = order[:min(K, Tb)]"),
    ("calibrate-centre-dropped", "            X = X - X.mean(axis=0, keepdims=True)",
     "            X = X"),
    ("calibrate-centre-per-head",
     "            X = X - X.mean(axis=0, keepdims=True)",
     "            X = (X.reshape(N, G, d) - X.reshape(N, G, d).mean(axis=0, keepdims=True)).reshape(N * G, d)"),
    ("residual-basis-smallest", "        order = np.argsort(-w, kind=\"stable\")[:r]\n        Vr = V[:, order]\n        for i in range(r):\n            j = int(np.argmax(np.abs(Vr[:, i])))\n            if Vr[j, i] < 0:\n                Vr[:, i] = -Vr[:, i]\n        U[kv] = Vr.astype(np.float32)\n    return U\n",
     "        order = np.argsort(w, kind=\"stable\")[:r]\n        Vr = V[:, order]\n        for i in range(r):\n            j = int(np.argmax(np.abs(Vr[:, i])))\n            if Vr[j, i] < 0:\n                Vr[:, i] = -Vr[:, i]\n        U[kv] = Vr.astype(np.float32)\n    return U\n"),
    ("key-mse-without-side-term", "        kh = kh + np.einsum(\"hdr,bhtr->bhtd\", np.asarray(U, np.float64), z)",
     "        kh = kh + 0.0 * np.einsum(\"hdr,bhtr->bhtd\", np.asarray(U, np.float64), z)"),
    ("channel-block-of-32", "KBLOCK = 64  # tokens per block of the per-channel base code",
     "KBLOCK = 32  # tokens per block of the per-channel base code"),
]

PINS = [
    ("test_base_code_hand_example", {}),
    ("test_base_code_two_groups_hand_example", {}),
    ("test_side_code_hand_example", {}),
    ("test_base_code_is_nearest_level", {"d": 64}),
    ("test_projection_exact_rational_sequential", {}),
    ("test_side_code_is_nearest_level", {"r": 16}),
    ("test_decode_brute_force_d8_T16", {}),
    ("test_sigma_zero_is_plain_base_code_attention", {}),
    ("test_unquantised_side_code_recovers_span_component", {}),
    ("test_kl_and_variance_against_library", {}),
    ("test_kl_direction_two_tokens", {}),
    ("test_lossless_limit_and_one_hot_value_distortion", {}),
    ("test_uniform_attention_value_distortion", {}),
    ("test_channel_code_hand_example", {}),
    ("test_channel_code_is_the_token_code_of_the_transpose", {}),
    ("test_channel_code_is_equivariant_to_a_shared_translation", {}),
    ("test_merge_of_token_shards_equals_whole", {}),
    ("test_a2_scores_sum_to_the_a2_diagnostic", {}),
    ("test_a2_scores_uniform_attention_closed_form", {}),
    ("test_a2_selection_minimises_the_surrogate_brute_force", {}),
    ("test_a2_mixed_values_limits", {}),
    ("test_calibration_centred_exact_rational", {}),
    ("test_calibration_centred_translation_and_library", {"i": 2}),
    ("test_residual_basis_is_the_residual_eigenbasis", {}),
    ("test_key_mse_pythagoras_and_lossless_limit", {}),
]


def _load_mutant(tmp_path, name, old, new, target="headq_oracle.c"):
    d = tmp_path / ("oracle_" + name.replace("-", "_"))
    d.mkdir()
    for f in ("__init__.py", "headq_oracle.c"):
        src = open(os.path.join(SRC_DIR, f)).read()
        if f == target:
            assert src.count(old) == 1, "mutation site not found exactly once: " + name
            src = src.replace(old, new)
        (d / f).write_text(src)
    modname = "oracle_mutant_" + uuid.uuid4().hex
    spec = importlib.util.spec_from_file_location(modname, str(d / "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    sys.modules[modname] = mod
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


ALL = [m + ("headq_oracle.c",) for m in MUTANTS] + [m + ("__init__.py",) for m in MUTANTS_PY]


@pytest.mark.parametrize("name,old,new,target", ALL, ids=[m[0] for m in ALL])
def test_pins_catch_mutant(tmp_path, monkeypatch, name, old, new, target):
    mod = _load_mutant(tmp_path, name, old, new, target)
    monkeypatch.setattr(pins, "oracle", mod)
    caught = []
    for fn, kw in PINS:
        try:
            getattr(pins, fn)(**kw)
        except Exception as exc:  # an assertion, or an error the slip provokes
            caught.append((fn, type(exc).__name__))
            break
    assert caught, "no pin caught the planted mistake '%s'" % name


def test_unmutated_copy_passes_every_pin(tmp_path, monkeypatch):
    mod = _load_mutant(tmp_path, "identity", "static int group_size(int d)",
                       "static int group_size(int d)")
    monkeypatch.setattr(pins, "oracle", mod)
    for fn, kw in PINS:
        getattr(pins, fn)(**kw)
