"""The product path and the oracle share no code and neither uses the other: no file of the
package (Python binding, build script, CUDA sources) imports, includes or names the oracle
module, and no file of the oracle imports the package."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "gated_deltanet_mixer_gdn_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _files(top, exts):
    for dirpath, _, names in os.walk(top):
        if "__pycache__" in dirpath:
            continue
        for n in names:
            if n.endswith(exts):
                yield os.path.join(dirpath, n)


def test_package_does_not_use_the_oracle():
    pat = re.compile(r"^\s*(import\s+oracle|from\s+oracle|#\s*include\s*[<\"].*oracle)", re.M)
    for f in _files(PKG, (".py", ".cu", ".cuh", ".h", ".c")):
        text = open(f, encoding="utf-8").read()
        assert not pat.search(text), f
        assert "oracle/" not in text and "libgdn_oracle" not in text and "gdn_oracle" not in text, f


def test_oracle_does_not_use_the_package():
    pat = re.compile(r"^\s*(import|from)\s+gated_deltanet_mixer_gdn_b200", re.M)
    for f in _files(ORACLE, (".py", ".c", ".h")):
        text = open(f, encoding="utf-8").read()
        assert not pat.search(text), f
        assert "gated_deltanet_mixer_gdn_b200" not in text and "libgdn_b200" not in text, f
