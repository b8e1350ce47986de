"""Builds libkda.so without importing the package (whose import loads the library).

``kda_build.build()`` runs gated_delta_rule_135_b200/build.py, loaded by file path, so a
fresh checkout (no library yet) or a stale library (built from older sources) can be
rebuilt before the package is imported.
"""
from __future__ import annotations

import importlib.util
import os

_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "gated_delta_rule_135_b200", "build.py")


def _module():
    spec = importlib.util.spec_from_file_location("_kda_library_build", _PATH)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def build(**kwargs) -> str:
    return _module().build(**kwargs)
