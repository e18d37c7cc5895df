"""The oracle: a plain float64 CPU implementation of the JEPA ViT encoder
forward.  Test infrastructure only -- the product path never imports it."""
