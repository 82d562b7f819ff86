from tree_verify_b200.build import build

print(build(force=True, verbose=True))
