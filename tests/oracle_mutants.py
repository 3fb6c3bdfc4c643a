"""Mutation check of the oracle's pins (test infrastructure, CPU only).

Plants one plausible mistake at a time in a scratch copy of ``oracle/`` and
runs the CPU oracle tests against it; every mistake must make some test fail.
One mutant is expected to survive and is reported as such:

* ``T8 fp32 division`` is equivalent: dividing the codebook's numerator and
  denominator in fp32 gives the same 127 magnitudes as the double division.

Usage:  python tests/oracle_mutants.py WORKDIR   (WORKDIR: an empty scratch
directory; the copy of oracle/ and the oracle tests is made there).
"""
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

EXPECTED_SURVIVORS = {"T8 fp32 division"}

# (file under oracle/, text to replace (must occur once), replacement, name)
MUTANTS = [
    ("nf4.py", "if abs(n - NF4[j]) < abs(n - NF4[best]):",
     "if abs(n - NF4[j]) <= abs(n - NF4[best]):", "encode_block ties to larger"),
    ("nf4.py", "scale = amax if amax else 1.0", "scale = amax if amax else 2.0",
     "encode_block zero-block scale"),
    ("nf4.py", "        n = v / scale\n", "        n = float(np.float32(v / scale))\n",
     "encode_block fp32 ratio"),
    ("nf4.py", "codes[b0:b0 + chunk_blocks] = np.argmin(dist, axis=2)",
     "codes[b0:b0 + chunk_blocks] = 15 - np.argmin(dist[:, :, ::-1], axis=2)",
     "quantize_nf4 ties to larger"),
    ("nf4.py", "scale = np.where(amax > 0, amax, 1.0)", "scale = np.where(amax > 0, amax, 0.5)",
     "quantize_nf4 zero-block scale"),
    ("nf4.py", "padded[:P] = w ", "padded[:P] = w * 1.0000001 ", "quantize_nf4 perturbed input"),
    ("nf4.py", "    padded = np.zeros(n1 * blocksize, dtype=np.float64)",
     "    padded = np.full(n1 * blocksize, 1e-30, dtype=np.float64)", "quantize_nf4 tail padding value"),
    ("nf4.py", "        n = blk / scale[:, None]                       # Python-double division",
     "        n = (blk / scale[:, None]).astype(np.float32).astype(np.float64)",
     "quantize_nf4 fp32 ratio"),
    ("nf4.py", "        amax[-1] = np.max(np.abs(w[full:]))", "        amax[-1] = np.max(np.abs(w[full - 1:]))",
     "block_scales ragged tail includes previous"),
    ("nf4.py", "payload = (c[0::2] << 4) | c[1::2]", "payload = (c[1::2] << 4) | c[0::2]",
     "pack low nibble first"),
    ("nf4.py", "PAD_CODE = 7 ", "PAD_CODE = 0 ", "pad code"),
    ("nf4.py", "codes[0::2] = payload >> 4\n    codes[1::2] = payload & 15",
     "codes[0::2] = payload & 15\n    codes[1::2] = payload >> 4", "unpack order"),
    ("nf4.py", "if length % 2 and (int(payload[-1]) & 15) != PAD_CODE:", "if False:",
     "unpack pad check dropped"),
    ("nf4.py", "    if length < 0 or payload.size != (length + 1) // 2:", "    if length < 0:",
     "unpack length check dropped"),
    ("nf4.py", "num = (1 << f) + 9 * (m + 1)", "num = (1 << f) + 9 * m", "T8 numerator"),
    ("nf4.py", "        e = 6 - f\n", "        e = 7 - f\n", "T8 exponent"),
    ("nf4.py", "out[u] = -mag if (u >> 7) else mag", "out[u] = mag", "T8 sign"),
    ("nf4.py", "mag = np.float32(num / den)", "mag = np.float32(np.float32(num) / np.float32(den))",
     "T8 fp32 division"),
    ("nf4.py", "if 2 * r > den or (2 * r == den and (N & 1)):", "if 2 * r >= den:",
     "mean rounding ties away"),
    ("nf4.py", "r = _round_rational_to_f32(total, v.size << 172)",
     "r = _round_rational_to_f32(total, (v.size + 1) << 172)", "mean divisor"),
    ("nf4.py", "total += s << int(ex - 24 + 172)", "total += s << int(ex - 23 + 172)",
     "mean exponent off by one"),
    ("nf4.py", "E = max(fl - 23, -149)", "E = max(fl - 22, -149)", "rational rounding precision"),
    ("nf4.py", "E = max(fl - 23, -149)", "E = max(fl - 23, -150)", "rational subnormal quantum"),
    ("nf4.py", "c = (a - offset).astype(np.float32)", "c = a.astype(np.float32)",
     "DQ no mean subtraction"),
    ("nf4.py", "s2[g] = mx if mx > 0 else np.float32(1.0)", "s2[g] = mx if mx > 0 else np.float32(0.5)",
     "DQ zero group scale"),
    ("nf4.py", "mx = np.max(np.abs(c[g * blocksize:(g + 1) * blocksize]))",
     "mx = np.max(np.abs(c[g * blocksize:max(g * blocksize + 1, (g + 1) * blocksize - 1)]))",
     "DQ group max misses last"),
    ("nf4.py", "code_of.setdefault(float(table[u]), u)", "code_of[float(table[u])] = u",
     "DQ zero code 0x80 instead of 0x00"),
    ("nf4.py", "d = np.abs(x[:, None] - values_sorted[None, :])\n    return np.argmin(d, axis=1)",
     "d = np.abs(x[:, None] - values_sorted[None, :])\n    return d.shape[1] - 1 - np.argmin(d[:, ::-1], axis=1)",
     "DQ ties to larger"),
    ("nf4.py", "        x = c[i0:i0 + chunk].astype(np.float64) / scale_el[i0:i0 + chunk]",
     "        x = (c[i0:i0 + chunk] / scale_el[i0:i0 + chunk].astype(np.float32)).astype(np.float64)",
     "DQ fp32 ratio"),
    ("nf4.py", "out = (t + np.float32(offset)).astype(np.float32)",
     "out = (t - np.float32(offset)).astype(np.float32)", "decode offset sign"),
    ("nf4.py", "g = np.arange(n1) // dq_blocksize",
     "g = np.minimum(np.arange(n1) // (dq_blocksize // 2), np.asarray(s2).size - 1)",
     "decode group index"),
    ("nf4.py", "    t = (table[q] * np.asarray(s2, dtype=np.float32)[g]).astype(np.float32)\n"
               "    out = (t + np.float32(offset)).astype(np.float32)",
     "    t = table[q].astype(np.float64) * np.asarray(s2, dtype=np.float64)[g]\n"
     "    out = (t + np.float64(offset)).astype(np.float32)", "decode fused"),
    ("nf4.py", "out[nz] = np.rint(x[nz] / quantum) * quantum",
     "out[nz] = np.floor(x[nz] / quantum) * quantum", "bf16 truncation"),
    ("nf4.py", "quantum = np.ldexp(1.0, np.maximum(e, -125) - 8)",
     "quantum = np.ldexp(1.0, np.maximum(e, -125) - 9)", "bf16 precision"),
    ("nf4.py", "quantum = np.ldexp(1.0, np.maximum(e, -125) - 8)",
     "quantum = np.ldexp(1.0, np.maximum(e, -126) - 8)", "bf16 subnormal threshold"),
    ("nf4.py", "    out[nz & (np.abs(out) > bf16_max)] = np.inf * np.sign(x[nz & (np.abs(out) > bf16_max)])\n",
     "", "bf16 overflow to inf dropped"),
    ("nf4.py", "per = a[np.arange(length) // blocksize]",
     "per = a[np.minimum((np.arange(length) + 1) // blocksize, a.size - 1)]",
     "dequant block index off by one"),
    ("nf4.py", "    if not np.all(np.isfinite(a)):\n        raise NonFiniteError(\"nonfinite reconstruction\")\n    per",
     "    per", "dequant nonfinite check dropped"),
    ("nf4.py", "return payload + 8 * n1 + 32 * n2 + 32", "return payload + 8 * n1 + 32 * n2",
     "bit budget offset"),
    ("linear.py", "Y = X @ W_hat + float(c) * (Z @ B)", "Y = X @ W_hat + (Z @ B)", "forward drops c"),
    ("linear.py", "    Z = X @ A\n    Y =",
     "    Z = (X.astype(np.float32) @ A.astype(np.float32)).astype(np.float64)\n    Y =",
     "forward Z in fp32"),
    ("linear.py", "dZ = c * (G @ B.T)", "dZ = (G @ B.T)", "dZ drops c"),
    ("linear.py", "dX = G @ W_hat.T + dZ @ A.T", "dX = G @ W_hat.T", "dX drops LoRA branch"),
    ("linear.py", "dX = G @ W_hat.T + dZ @ A.T", "dX = G @ W_hat.T - dZ @ A.T", "dX sign"),
    ("linear.py", "dX = G @ W_hat.T + dZ @ A.T", "dX = G @ W_hat.T + dZ @ A.T * (1 + 1e-6)",
     "dX LoRA branch scaled 1e-6"),
    ("linear.py", "dA = X.T @ dZ", "dA = X.T @ (G @ B.T)", "dA drops c"),
    ("linear.py", "dB = c * (Z.T @ G)", "dB = (Z.T @ G)", "dB drops c"),
    ("linear.py", "    Z = X @ A\n    dZ", "    Z = X @ (A * (1 + 2**-20))\n    dZ", "backward Z perturbed"),
    ("merge.py", "return W_hat + float(c) * (A @ B)", "return W_hat + (A @ B)", "merge drops c"),
    ("merge.py", "return W_hat + float(c) * (A @ B)",
     "return W_hat + float(c) * (A @ B).astype(np.float32)", "merge product in fp32"),
    ("merge.py", "return round_to_bf16(merge_exact(W_hat, A, B, c))",
     "return merge_exact(W_hat, A, B, c)", "merge no rounding"),
    ("int4.py", "r = math.floor(abs(t) + 0.5) * (1 if t >= 0 else -1)", "r = round(t)",
     "int4 ties to even"),
    ("int4.py", "s = amax / 7.0 if amax else 1.0", "s = amax / 8.0 if amax else 1.0", "int4 scale"),
    ("int4.py", "codes = (q + 8).astype(np.uint8).ravel()[:n]",
     "codes = (q + 7).astype(np.uint8).ravel()[:n]", "int4 code offset"),
    ("int4.py", "s = np.where(amax > 0, amax / 7.0, 1.0).astype(np.float32)",
     "s = np.where(amax > 0, (amax / 7.0).astype(np.float32).astype(np.float64) * (1 + 2**-20), 1.0).astype(np.float32)",
     "int4 stored scale rounding"),
    ("int4.py", "    xb = np.concatenate([x, np.zeros(pad)]).reshape(n1, blocksize)",
     "    xb = np.concatenate([x, np.full(pad, 1e-3)]).reshape(n1, blocksize)", "int4 tail padding value"),
    ("int4.py", "per = s[np.arange(c.size) // blocksize]",
     "per = s[np.minimum((np.arange(c.size) + 1) // blocksize, s.size - 1)]", "int4 dequant block index"),
    ("int4.py", "return round_to_bf16((c - 8) * per)", "return (c - 8) * per", "int4 dequant no bf16"),
]


def _copy(work):
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(work, "oracle"))
    os.makedirs(os.path.join(work, "tests"))
    for f in os.listdir(os.path.join(ROOT, "tests")):
        if (f.startswith("test_oracle") and "mutants" not in f) or f == "conftest.py":
            shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(work, "tests", f))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(work, "tests", "golden"))


def _run(work):
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(work, "tests"), "-x", "-q",
                        "-p", "no:cacheprovider", "-m", "not gpu"],
                       capture_output=True, text=True, cwd=work)
    return r.returncode == 0


def main():
    if len(sys.argv) != 2:
        print(__doc__)
        return 2
    work = os.path.abspath(sys.argv[1])
    if os.path.exists(work) and os.listdir(work):
        print(f"{work} is not empty")
        return 2
    os.makedirs(work, exist_ok=True)
    _copy(work)
    if not _run(work):
        print("the unmodified oracle fails its tests")
        return 1
    unexpected = []
    for fn, old, new, name in MUTANTS:
        path = os.path.join(work, "oracle", fn)
        src = open(path).read()
        assert src.count(old) == 1, (name, old)
        open(path, "w").write(src.replace(old, new))
        survived = _run(work)
        open(path, "w").write(src)
        tag = "survived (expected)" if survived and name in EXPECTED_SURVIVORS else \
              "SURVIVED" if survived else "killed"
        print(f"{tag:20s} {name}")
        if survived and name not in EXPECTED_SURVIVORS:
            unexpected.append(name)
    print(f"{len(MUTANTS)} mutants, unexpected survivors: {unexpected}")
    return 1 if unexpected else 0


if __name__ == "__main__":
    sys.exit(main())
