"""The product path and the oracle stay apart: nothing in the package or the C ABI
headers names, imports or links the oracle, and the oracle shares no source with the
CUDA path (only tests, the smoke check and the bench's CPU baseline use it)."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PRODUCT = [os.path.join(ROOT, "differential_latent_attention_b200"), os.path.join(ROOT, "include")]
SOURCE = (".py", ".cu", ".cuh", ".h", ".c", ".cpp")


def _files(dirs):
    for d in dirs:
        for base, _, names in os.walk(d):
            for n in names:
                if n.endswith(SOURCE):
                    yield os.path.join(base, n)


def test_product_never_names_the_oracle():
    hits = [f for f in _files(PRODUCT) if re.search(r"\boracle\b", open(f, errors="replace").read())]
    assert not hits, hits


def test_oracle_includes_no_product_header():
    oracle_dir = os.path.join(ROOT, "oracle")
    src = "".join(open(f).read() for f in _files([oracle_dir]))
    included = set(re.findall(r'#include\s+"([^"]+)"', src))
    product_headers = {os.path.basename(f) for f in _files(PRODUCT) if f.endswith((".h", ".cuh"))}
    assert not (included & product_headers), included & product_headers
    assert "differential_latent_attention_b200" not in src
