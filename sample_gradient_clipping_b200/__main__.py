from .build import build

build(force=True, verbose=True)
