"""libbha: block-hybrid attention (softmax inside the active block, Hedgehog linear
attention across committed blocks) for blockwise diffusion-LM decoding on B200."""
