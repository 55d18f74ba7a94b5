"""Test helper: build libsana.so if needed and import the binding."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from softmax_attention_sana_b200 import build as _build  # noqa: E402

_build.build()

import softmax_attention_sana_b200 as sana  # noqa: E402,F401
from softmax_attention_sana_b200 import _lib  # noqa: E402,F401
